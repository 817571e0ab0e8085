"""B200-native paged KV-cache decode attention.

The compute path lives in ``libpkv.so`` (CUDA for sm_100a plus the host block
allocator, behind the C ABI declared in ``include/pkv.h``).  ``pkv`` is the
thin ctypes binding over it, imported on first use.
"""
from importlib import import_module as _import_module

__all__ = ["pkv"]


def __getattr__(name):
    if name in __all__:
        return _import_module(f"{__name__}.{name}")
    if name in ("paged_kv_write", "paged_attention_decode", "BlockAllocator"):
        return getattr(_import_module(f"{__name__}.pkv"), name)
    raise AttributeError(name)
