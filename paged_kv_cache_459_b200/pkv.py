"""Python binding of libpkv.so (ctypes): argument marshalling only.

Every step of the path runs in the library's CUDA kernels; PyTorch supplies
device memory and the current stream.  If the library has not been built the
import fails loudly -- there is no fallback implementation.

    paged_kv_write(k, v, k_cache, v_cache, slot_mapping)
    paged_attention_decode(out, q, k_cache, v_cache, block_tables, seq_lens, scale, num_kv_heads)
    BlockAllocator(num_blocks, free_order=None)   # host allocator (C++)
"""
from __future__ import annotations

import ctypes
import os
import re

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpkv.so")
HEADER = os.path.join(os.path.dirname(_HERE), "include", "pkv.h")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m paged_kv_cache_459_b200.build` "
        "(nvcc, sm_100a). There is no CPU fallback.")

_lib = ctypes.CDLL(LIB_PATH)

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_OOM, ERR_CUDA = range(6)
DEV_ERR_BAD_SLOT, DEV_ERR_BAD_BLOCK, DEV_ERR_BAD_LEN, DEV_ERR_TIMEOUT = 1, 2, 4, 8
DECODE_AUTO, DECODE_SINGLE, DECODE_SPLIT, DECODE_CLUSTER = 0, 1, 2, 4
SWAP_OUT, SWAP_IN = 0, 1
BLOCK_TOKENS = 16
DEFAULT_PARTITION_TOKENS = 512

_P, _i32, _i64, _f32, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
_sigs = {
    "pkv_status_string": ([_i32], ctypes.c_char_p),
    "pkv_last_cuda_error": ([], _i32),
    "pkv_last_cuda_error_string": ([], ctypes.c_char_p),
    "pkv_block_tokens": ([], _i32),
    "pkv_version": ([], ctypes.c_char_p),
    "pkv_paged_kv_write": ([_P, _P, _P, _P, _P, _i32, _i32, _i32, _i64, _P, _P], _i32),
    "pkv_decode_workspace_bytes": ([_i32, _i32, _i32, _i32, _i32], _sz),
    "pkv_decode_workspace_bytes_for": ([_i32, _i32, _i32, _i32, _i32, _i32, _i32], _sz),
    "pkv_decode_variant_for": ([_i32, _i32, _i32, _i32, _i32, _i32, _sz], _i32),
    "pkv_decode_cluster_parts_for": ([_i32, _i32, _i32, _i32, _i32, _i32, _i32, _sz], _i32),
    "pkv_paged_attention_decode": ([_P, _P, _P, _P, _P, _i32, _P, _i32, _i32, _i32, _i32, _i64,
                                    _f32, _P, _sz, _P, _P], _i32),
    "pkv_paged_attention_decode_ex": ([_P, _P, _P, _P, _P, _i32, _P, _i32, _i32, _i32, _i32, _i64,
                                       _f32, _i32, _i32, _P, _sz, _P, _P], _i32),
    "pkv_paged_attention_decode_static": ([_P, _P, _P, _P, _P, _i32, _P, _i32, _i32, _i32, _i32,
                                           _i64, _f32, _i32, _P, _P], _i32),
    "pkv_alloc_create": ([_i64, _P, _P], _i32),
    "pkv_alloc_destroy": ([_P], None),
    "pkv_alloc_add_seq": ([_P, _i64, _i64], _i32),
    "pkv_alloc_fork": ([_P, _i64, _i64, _i64], _i32),
    "pkv_alloc_append_token": ([_P, _i64, _P], _i32),
    "pkv_alloc_append_tokens": ([_P, _P, _i32, _P], _i32),
    "pkv_alloc_append_tokens_into": ([_P, _P, _i32, _P, _i32, _P, _P], _i32),
    "pkv_alloc_free_seq": ([_P, _i64], _i32),
    "pkv_alloc_export": ([_P, _P, _i32, _i32, _P, _P], _i32),
    "pkv_alloc_stats": ([_P, _P, _P, _P, _P], _i32),
    "pkv_alloc_free_list": ([_P, _P, _i64, _P], _i32),
    "pkv_alloc_refcount": ([_P, _i64, _P], _i32),
    "pkv_alloc_take_copies": ([_P, _P, _P, _i64, _P], _i32),
    "pkv_copy_blocks": ([_P, _P, _P, _P, _i32, _i32, _i32, _i64, _P, _P], _i32),
    "pkv_swap_blocks": ([_P, _P, _P, _P, _P, _P, _i32, _i32, _i32, _i32, _i64, _i64, _P, _P], _i32),
    "pkv_alloc_set_host_pool": ([_P, _i64], _i32),
    "pkv_alloc_extend": ([_P, _i64, _i64, _P], _i32),
    "pkv_paged_attention_prefill": ([_P, _P, _P, _P, _P, _i32, _P, _P, _i32, _i32, _i32, _i32, _i32,
                                     _i64, _f32, _P, _P], _i32),
    "pkv_alloc_swap_out": ([_P, _i64], _i32),
    "pkv_alloc_swap_in": ([_P, _i64], _i32),
    "pkv_alloc_take_swaps": ([_P, _i32, _P, _P, _i64, _P], _i32),
    "pkv_alloc_prefix_groups": ([_P, _P, _i32, _P, _P, _P, _P], _i32),
    "pkv_decode_prefix_workspace_bytes": ([_i32, _i32, _i32, _i32, _i32], _sz),
    "pkv_paged_decode_step": ([_P, _P, _P, _P, _P, _P, _P, _i32, _P, _i32, _i32, _i32, _i32, _i64,
                               _f32, _i32, _i32, _P, _sz, _P, _P], _i32),
    "pkv_paged_decode_prefix_step": ([_P, _P, _P, _P, _P, _P, _P, _i32, _P, _i32, _i32, _i32, _i32,
                                      _i64, _f32, _P, _P, _P, _i32, _i32, _i32, _P, _sz, _P, _P],
                                     _i32),
    "pkv_paged_attention_decode_prefix": ([_P, _P, _P, _P, _P, _i32, _P, _i32, _i32, _i32, _i32,
                                           _i64, _f32, _P, _P, _P, _i32, _i32, _i32, _P, _sz, _P,
                                           _P],
                                          _i32),
    "pkv_alloc_seq_len": ([_P, _i64, _P], _i32),
    "pkv_alloc_slot_of": ([_P, _i64, _i64, _P], _i32),
}
for _name, (_args, _res) in _sigs.items():
    _fn = getattr(_lib, _name)
    _fn.argtypes = _args
    _fn.restype = _res


def lib() -> ctypes.CDLL:
    return _lib


def declared_symbols(header: str = HEADER) -> list[str]:
    """Names of the functions include/pkv.h declares."""
    text = open(header).read()
    return sorted(set(re.findall(r"^PKV_API[^(;]*?\b(pkv_\w+)\s*\(", text, flags=re.M)))


def status_string(code: int) -> str:
    return _lib.pkv_status_string(code).decode()


class PkvError(RuntimeError):
    def __init__(self, code: int, what: str):
        msg = f"{what}: {status_string(code)} ({code})"
        if code == ERR_CUDA and _lib.pkv_last_cuda_error():
            msg += f": {_lib.pkv_last_cuda_error_string().decode()}"
        super().__init__(msg)
        self.code = code


def _check(code: int, what: str) -> None:
    if code != OK:
        raise PkvError(code, what)


# ------------------------------------------------------------------ kernels
def _dev_tensor(t, dtype, name):
    import torch

    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be on a CUDA device")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _stream_ptr(device) -> int:
    import torch

    return torch.cuda.current_stream(device).cuda_stream


def paged_kv_write(k, v, k_cache, v_cache, slot_mapping, err=None) -> None:
    """k, v [T, Hkv, d] bf16; caches [NB, Hkv, 16, d] bf16; slot_mapping [T] int64."""
    import torch

    bf = torch.bfloat16
    T, hkv, d = k.shape
    if v.shape != k.shape or k_cache.shape != v_cache.shape or k_cache.dim() != 4 \
            or tuple(k_cache.shape[1:]) != (hkv, BLOCK_TOKENS, d) or slot_mapping.shape != (T,):
        raise ValueError("shape mismatch")
    ptrs = [_dev_tensor(x, bf, n) for x, n in ((k, "k"), (v, "v"), (k_cache, "k_cache"),
                                                 (v_cache, "v_cache"))]
    sp = _dev_tensor(slot_mapping, torch.int64, "slot_mapping")
    ep = _dev_tensor(err, torch.int32, "err") if err is not None else None
    _check(_lib.pkv_paged_kv_write(*ptrs, sp, T, hkv, d, k_cache.shape[0], ep,
                                   _stream_ptr(k.device)), "pkv_paged_kv_write")


def copy_blocks(k_cache, v_cache, src, dst, err=None) -> None:
    """Copy whole blocks src[i] -> dst[i] (device int64) in both caches."""
    import torch

    if k_cache.shape != v_cache.shape or k_cache.dim() != 4 or src.shape != dst.shape:
        raise ValueError("shape mismatch")
    nb, hkv, bt, d = k_cache.shape
    ptrs = [_dev_tensor(x, torch.bfloat16, n) for x, n in ((k_cache, "k_cache"), (v_cache, "v_cache"))]
    sp = _dev_tensor(src, torch.int64, "src")
    dp = _dev_tensor(dst, torch.int64, "dst")
    ep = _dev_tensor(err, torch.int32, "err") if err is not None else None
    _check(_lib.pkv_copy_blocks(*ptrs, sp, dp, src.numel(), hkv, d, nb, ep,
                                _stream_ptr(k_cache.device)), "pkv_copy_blocks")


def swap_blocks(k_cache, v_cache, host_k, host_v, gpu_blocks, host_blocks, direction,
                err=None) -> None:
    """Move whole blocks between the GPU caches and pinned host swap space
    (host_k/host_v: pinned CPU bf16 tensors [num_host_blocks, Hkv, 16, d])."""
    import torch

    if k_cache.shape != v_cache.shape or host_k.shape != host_v.shape \
            or tuple(host_k.shape[1:]) != tuple(k_cache.shape[1:]) \
            or gpu_blocks.shape != host_blocks.shape:
        raise ValueError("shape mismatch")
    for t, n in ((host_k, "host_k"), (host_v, "host_v")):
        if t.device.type != "cpu" or not t.is_pinned() or t.dtype != torch.bfloat16 \
                or not t.is_contiguous():
            raise ValueError(f"{n} must be a pinned, contiguous bf16 CPU tensor")
    nb, hkv, bt, d = k_cache.shape
    ptrs = [_dev_tensor(x, torch.bfloat16, n) for x, n in ((k_cache, "k_cache"), (v_cache, "v_cache"))]
    gp = _dev_tensor(gpu_blocks, torch.int64, "gpu_blocks")
    hp = _dev_tensor(host_blocks, torch.int64, "host_blocks")
    ep = _dev_tensor(err, torch.int32, "err") if err is not None else None
    _check(_lib.pkv_swap_blocks(*ptrs, host_k.data_ptr(), host_v.data_ptr(), gp, hp,
                                gpu_blocks.numel(), int(direction), hkv, d, nb, host_k.shape[0], ep,
                                _stream_ptr(k_cache.device)), "pkv_swap_blocks")


def paged_attention_prefill(out, q, k_cache, v_cache, block_tables, seq_lens, query_start, scale,
                            num_kv_heads, max_query_len: int, err=None) -> None:
    """Causal attention of each sequence's new tokens over its paged K/V.
    q, out [T, Hq, d] bf16; query_start [B + 1] int32 (rows of each sequence);
    seq_lens [B] int32 context lengths including the new tokens."""
    import torch

    T, hq, d = q.shape
    B = seq_lens.shape[0]
    if out.shape != q.shape or k_cache.shape != v_cache.shape or k_cache.dim() != 4 \
            or tuple(k_cache.shape[1:]) != (num_kv_heads, BLOCK_TOKENS, d) \
            or block_tables.shape[0] != B or query_start.shape != (B + 1,):
        raise ValueError("shape mismatch")
    ptrs = [_dev_tensor(x, torch.bfloat16, n) for x, n in ((out, "out"), (q, "q"),
                                                            (k_cache, "k_cache"),
                                                            (v_cache, "v_cache"))]
    tp = _dev_tensor(block_tables, torch.int32, "block_tables")
    lp = _dev_tensor(seq_lens, torch.int32, "seq_lens")
    sp = _dev_tensor(query_start, torch.int32, "query_start")
    ep = _dev_tensor(err, torch.int32, "err") if err is not None else None
    _check(_lib.pkv_paged_attention_prefill(*ptrs, tp, block_tables.shape[1], lp, sp, B,
                                            int(max_query_len), hq, num_kv_heads, d,
                                            k_cache.shape[0], float(scale), ep,
                                            _stream_ptr(q.device)), "pkv_paged_attention_prefill")


_workspaces: dict = {}


def _workspace(device, nbytes: int):
    import torch

    key = (device.type, device.index)
    ws = _workspaces.get(key)
    if ws is None or ws.numel() < nbytes:
        ws = torch.empty(max(nbytes, 1 << 20), dtype=torch.uint8, device=device)
        _workspaces[key] = ws
    return ws


def decode_workspace_bytes(num_seqs, num_heads, head_dim, max_blocks_per_seq,
                           partition_tokens=DEFAULT_PARTITION_TOKENS) -> int:
    return int(_lib.pkv_decode_workspace_bytes(num_seqs, num_heads, head_dim, max_blocks_per_seq,
                                               partition_tokens))


def decode_workspace_bytes_for(variant, num_seqs, num_heads, num_kv_heads, head_dim,
                               max_blocks_per_seq,
                               partition_tokens=DEFAULT_PARTITION_TOKENS) -> int:
    return int(_lib.pkv_decode_workspace_bytes_for(variant, num_seqs, num_heads, num_kv_heads,
                                                   head_dim, max_blocks_per_seq, partition_tokens))


def decode_variant_for(num_seqs, num_heads, num_kv_heads, head_dim, max_blocks_per_seq,
                       partition_tokens=DEFAULT_PARTITION_TOKENS, workspace_bytes=0) -> int:
    """The variant the automatic choice takes for these sizes and workspace."""
    return int(_lib.pkv_decode_variant_for(num_seqs, num_heads, num_kv_heads, head_dim,
                                           max_blocks_per_seq, partition_tokens, workspace_bytes))


def decode_cluster_parts_for(num_seqs, num_heads, num_kv_heads, head_dim, max_blocks_per_seq,
                             variant=DECODE_AUTO, partition_tokens=DEFAULT_PARTITION_TOKENS,
                             workspace_bytes=0) -> int:
    """Parts per sequence of the cluster variant for these sizes (0 when the
    variant does not run as the cluster variant)."""
    return int(_lib.pkv_decode_cluster_parts_for(num_seqs, num_heads, num_kv_heads, head_dim,
                                                 max_blocks_per_seq, variant, partition_tokens,
                                                 workspace_bytes))


def _decode_args(out, q, new_kv, k_cache, v_cache, block_tables, seq_lens, num_kv_heads, variant,
                 partition_tokens, workspace, err):
    """Checked pointers and sizes shared by the decode entry points: (out, q,
    [k_new, v_new,] k_cache, v_cache) then the table / length / size arguments
    up to num_blocks, and (workspace, bytes, err)."""
    import torch

    B, hq, d = q.shape
    W = block_tables.shape[1] if block_tables.dim() == 2 else -1
    if out.shape != q.shape or k_cache.shape != v_cache.shape or k_cache.dim() != 4 \
            or tuple(k_cache.shape[1:]) != (num_kv_heads, BLOCK_TOKENS, d) \
            or block_tables.dim() != 2 or block_tables.shape[0] != B or seq_lens.shape != (B,) \
            or any(x.shape != (B, num_kv_heads, d) for x in new_kv):
        raise ValueError("shape mismatch")
    named = [(out, "out"), (q, "q")] + list(zip(new_kv, ("k_new", "v_new"))) + \
        [(k_cache, "k_cache"), (v_cache, "v_cache")]
    ptrs = [_dev_tensor(x, torch.bfloat16, n) for x, n in named]
    sizes = [_dev_tensor(block_tables, torch.int32, "block_tables"), W,
             _dev_tensor(seq_lens, torch.int32, "seq_lens"), B, hq, num_kv_heads, d,
             k_cache.shape[0]]
    need = decode_workspace_bytes_for(variant, B, hq, num_kv_heads, d, W, partition_tokens) \
        if W > 0 and num_kv_heads > 0 and hq % num_kv_heads == 0 else 0
    if workspace is None and need > 0:
        workspace = _workspace(q.device, need)
    tail = [_dev_tensor(workspace, torch.uint8, "workspace") if workspace is not None else None,
            workspace.numel() if workspace is not None else 0,
            _dev_tensor(err, torch.int32, "err") if err is not None else None]
    return ptrs, sizes, tail


def paged_attention_decode(out, q, k_cache, v_cache, block_tables, seq_lens, scale, num_kv_heads,
                           *, variant: int = DECODE_AUTO,
                           partition_tokens: int = DEFAULT_PARTITION_TOKENS,
                           workspace=None, err=None) -> None:
    """out, q [B, Hq, d] bf16; caches [NB, Hkv, 16, d] bf16; block_tables [B, W]
    int32; seq_lens [B] int32.  The split-K workspace is allocated once per
    device and reused unless one is passed in (a uint8 CUDA tensor)."""
    ptrs, sizes, tail = _decode_args(out, q, (), k_cache, v_cache, block_tables, seq_lens,
                                     num_kv_heads, variant, partition_tokens, workspace, err)
    _check(_lib.pkv_paged_attention_decode_ex(*ptrs, *sizes, float(scale), variant,
                                              partition_tokens, *tail, _stream_ptr(q.device)),
           "pkv_paged_attention_decode")


def paged_decode_step(out, q, k_new, v_new, k_cache, v_cache, block_tables, seq_lens, scale,
                      num_kv_heads, *, variant: int = DECODE_AUTO,
                      partition_tokens: int = DEFAULT_PARTITION_TOKENS,
                      workspace=None, err=None) -> None:
    """The write of k_new / v_new [B, Hkv, d] (each sequence's new token, at
    position seq_lens[b] - 1) fused into paged_attention_decode: one call for
    the whole step (see include/pkv.h, pkv_paged_decode_step)."""
    ptrs, sizes, tail = _decode_args(out, q, (k_new, v_new), k_cache, v_cache, block_tables,
                                     seq_lens, num_kv_heads, variant, partition_tokens, workspace,
                                     err)
    _check(_lib.pkv_paged_decode_step(*ptrs, *sizes, float(scale), variant, partition_tokens,
                                      *tail, _stream_ptr(q.device)),
           "pkv_paged_decode_step")


class PreparedDecodeStep:
    """paged_decode_step bound to fixed tensors: the checks and the pointer
    marshalling run once, here; each call passes the stored pointers and
    the current stream to pkv_paged_decode_step.  For serving loops that
    reuse the same device buffers every step (the tensors must stay alive
    and keep their shapes; their contents may change between calls)."""

    def __init__(self, out, q, k_new, v_new, k_cache, v_cache, block_tables, seq_lens, scale,
                 num_kv_heads, *, variant: int = DECODE_AUTO,
                 partition_tokens: int = DEFAULT_PARTITION_TOKENS, workspace=None, err=None):
        ptrs, sizes, tail = _decode_args(out, q, (k_new, v_new), k_cache, v_cache, block_tables,
                                         seq_lens, num_kv_heads, variant, partition_tokens,
                                         workspace, err)
        self._keep = (out, q, k_new, v_new, k_cache, v_cache, block_tables, seq_lens, workspace,
                      err, _workspaces.get((q.device.type, q.device.index)))
        self._args = (*ptrs, *sizes, float(scale), variant, partition_tokens, *tail)
        self._device = q.device
        self._fn = _lib.pkv_paged_decode_step

    def __call__(self) -> None:
        code = self._fn(*self._args, _stream_ptr(self._device))
        if code != OK:
            raise PkvError(code, "pkv_paged_decode_step")


def prepare_decode_step(out, q, k_new, v_new, k_cache, v_cache, block_tables, seq_lens, scale,
                        num_kv_heads, **kw) -> PreparedDecodeStep:
    """A PreparedDecodeStep: paged_decode_step with its argument checks done once."""
    return PreparedDecodeStep(out, q, k_new, v_new, k_cache, v_cache, block_tables, seq_lens,
                              scale, num_kv_heads, **kw)


def decode_prefix_workspace_bytes(num_seqs, num_heads, head_dim, max_blocks_per_seq,
                                  partition_tokens=DEFAULT_PARTITION_TOKENS) -> int:
    return int(_lib.pkv_decode_prefix_workspace_bytes(num_seqs, num_heads, head_dim,
                                                      max_blocks_per_seq, partition_tokens))


def _prefix_args(out, q, new_kv, k_cache, v_cache, block_tables, seq_lens, num_kv_heads,
                 prefix_blocks, group_offsets, group_seqs, partition_tokens, workspace, err):
    """Checked pointers and sizes shared by the cascade entry points: (out, q,
    [k_new, v_new,] k_cache, v_cache), the table / length / size arguments up
    to num_blocks, the group arrays, and (workspace, bytes, err)."""
    import torch

    B, hq, d = q.shape
    W = block_tables.shape[1]
    if out.shape != q.shape or k_cache.shape != v_cache.shape or k_cache.dim() != 4 \
            or tuple(k_cache.shape[1:]) != (num_kv_heads, BLOCK_TOKENS, d) \
            or block_tables.shape[0] != B or seq_lens.shape != (B,) or prefix_blocks.shape != (B,) \
            or any(x.shape != (B, num_kv_heads, d) for x in new_kv):
        raise ValueError("shape mismatch")
    named = [(out, "out"), (q, "q")] + list(zip(new_kv, ("k_new", "v_new"))) + \
        [(k_cache, "k_cache"), (v_cache, "v_cache")]
    ptrs = [_dev_tensor(x, torch.bfloat16, n) for x, n in named]
    sizes = [_dev_tensor(block_tables, torch.int32, "block_tables"), W,
             _dev_tensor(seq_lens, torch.int32, "seq_lens"), B, hq, num_kv_heads, d,
             k_cache.shape[0]]
    groups = [_dev_tensor(prefix_blocks, torch.int32, "prefix_blocks"),
              _dev_tensor(group_offsets, torch.int32, "group_offsets"),
              _dev_tensor(group_seqs, torch.int32, "group_seqs") if group_seqs.numel() else None,
              group_offsets.numel() - 1]
    if workspace is None:
        workspace = _workspace(q.device, decode_prefix_workspace_bytes(B, hq, d, W,
                                                                       partition_tokens))
    tail = [_dev_tensor(workspace, torch.uint8, "workspace"), workspace.numel(),
            _dev_tensor(err, torch.int32, "err") if err is not None else None]
    return ptrs, sizes, groups, tail


def paged_attention_decode_prefix(out, q, k_cache, v_cache, block_tables, seq_lens, scale,
                                  num_kv_heads, prefix_blocks, group_offsets, group_seqs, *,
                                  max_suffix_blocks: int = 0,
                                  partition_tokens: int = DEFAULT_PARTITION_TOKENS,
                                  workspace=None, err=None) -> None:
    """Decode with shared prefixes read once per group (see include/pkv.h).
    prefix_blocks [B], group_offsets [G + 1], group_seqs [members]: int32 CUDA.
    max_suffix_blocks: bound on the blocks past each prefix (0: unknown);
    suffix_blocks_bound() computes it from host arrays."""
    ptrs, sizes, groups, tail = _prefix_args(out, q, (), k_cache, v_cache, block_tables, seq_lens,
                                             num_kv_heads, prefix_blocks, group_offsets,
                                             group_seqs, partition_tokens, workspace, err)
    _check(_lib.pkv_paged_attention_decode_prefix(*ptrs, *sizes, float(scale), *groups,
                                                  int(max_suffix_blocks), partition_tokens,
                                                  *tail, _stream_ptr(q.device)),
           "pkv_paged_attention_decode_prefix")


def paged_decode_prefix_step(out, q, k_new, v_new, k_cache, v_cache, block_tables, seq_lens, scale,
                             num_kv_heads, prefix_blocks, group_offsets, group_seqs, *,
                             max_suffix_blocks: int = 0,
                             partition_tokens: int = DEFAULT_PARTITION_TOKENS,
                             workspace=None, err=None) -> None:
    """paged_attention_decode_prefix with the write of k_new / v_new [B, Hkv, d]
    (each sequence's new token, at position seq_lens[b] - 1) fused in."""
    ptrs, sizes, groups, tail = _prefix_args(out, q, (k_new, v_new), k_cache, v_cache,
                                             block_tables, seq_lens, num_kv_heads, prefix_blocks,
                                             group_offsets, group_seqs, partition_tokens,
                                             workspace, err)
    _check(_lib.pkv_paged_decode_prefix_step(*ptrs, *sizes, float(scale), *groups,
                                             int(max_suffix_blocks), partition_tokens, *tail,
                                             _stream_ptr(q.device)),
           "pkv_paged_decode_prefix_step")


def suffix_blocks_bound(seq_lens, prefix_blocks) -> int:
    """max over the batch of ceil(len / 16) - prefix_blocks (host arrays): the
    max_suffix_blocks argument of paged_attention_decode_prefix."""
    lens = np.asarray(seq_lens, dtype=np.int64)
    pb = np.asarray(prefix_blocks, dtype=np.int64)
    if lens.size == 0:
        return 0
    return int(max(1, (-(-lens // BLOCK_TOKENS) - pb).max()))


# ---------------------------------------------------------------- allocator
class AllocError(PkvError):
    @property
    def kind(self) -> str:
        return {ERR_OOM: "oom", ERR_UNSUPPORTED: "unsupported"}.get(self.code, "invalid")


def _addr(a: np.ndarray) -> int:
    """Address of a C-contiguous array's data: the per-step allocator calls
    take it this way (about half the cost of a.ctypes.data), falling back to
    a.ctypes.data for read-only or empty arrays."""
    try:
        return ctypes.addressof(ctypes.c_char.from_buffer(a))
    except (TypeError, ValueError, BufferError):
        return a.ctypes.data


def _acheck(code: int, what: str) -> None:
    if code != OK:
        raise AllocError(code, what)


class BlockAllocator:
    """The C++ block allocator: reference-counted blocks, per-sequence tables."""

    def __init__(self, num_blocks: int, free_order=None):
        h = ctypes.c_void_p()
        order = None
        if free_order is not None:
            order = np.ascontiguousarray(free_order, dtype=np.int64)
            if order.shape != (num_blocks,):
                raise AllocError(ERR_INVALID_ARG, "free order length")
        _acheck(_lib.pkv_alloc_create(int(num_blocks), order.ctypes.data if order is not None
                                      else None, ctypes.byref(h)), "pkv_alloc_create")
        self._h = h
        self._destroy = _lib.pkv_alloc_destroy  # kept: module globals may be gone at exit
        self.num_blocks = int(num_blocks)

    def __del__(self):
        h = getattr(self, "_h", None)
        if h is not None and h.value:
            self._destroy(h)
            self._h = None

    def add_seq(self, seq_id: int, num_tokens: int) -> None:
        _acheck(_lib.pkv_alloc_add_seq(self._h, int(seq_id), int(num_tokens)), "add_seq")

    def fork(self, parent: int, child: int, num_tokens: int | None = None) -> None:
        _acheck(_lib.pkv_alloc_fork(self._h, int(parent), int(child),
                                    -1 if num_tokens is None else int(num_tokens)), "fork")

    def append_token(self, seq_id: int) -> int:
        out = ctypes.c_int64()
        _acheck(_lib.pkv_alloc_append_token(self._h, int(seq_id), ctypes.byref(out)), "append_token")
        return out.value

    def extend(self, seq_id: int, n: int) -> np.ndarray:
        """Slots of n more tokens (blocks taken as each fills)."""
        out = np.empty(int(n), dtype=np.int64)
        _acheck(_lib.pkv_alloc_extend(self._h, int(seq_id), int(n),
                                      out.ctypes.data if n else None), "extend")
        return out

    def append_tokens(self, seq_ids) -> np.ndarray:
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        out = np.empty(len(ids), dtype=np.int64)
        _acheck(_lib.pkv_alloc_append_tokens(self._h, _addr(ids), len(ids), _addr(out)),
                "append_tokens")
        return out

    def append_tokens_into(self, seq_ids, tables: np.ndarray, lens: np.ndarray) -> np.ndarray:
        """append_tokens, with the host tables / lengths that export() gave for
        the same seq_ids updated in place (only the entries the step changes)."""
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        n = len(ids)
        if (not isinstance(tables, np.ndarray) or tables.dtype != np.int32 or tables.ndim != 2
                or tables.shape[0] != n or tables.shape[1] < 1 or not tables.flags.c_contiguous
                or not tables.flags.writeable or not isinstance(lens, np.ndarray)
                or lens.dtype != np.int32 or lens.shape != (n,) or not lens.flags.c_contiguous
                or not lens.flags.writeable):
            raise AllocError(ERR_INVALID_ARG, "append_tokens_into: tables int32 [n][width] and "
                                              "lens int32 [n], C-contiguous and writeable")
        out = np.empty(n, dtype=np.int64)
        _acheck(_lib.pkv_alloc_append_tokens_into(self._h, _addr(ids), n, _addr(out),
                                                  int(tables.shape[1]), _addr(tables), _addr(lens)),
                "append_tokens_into")
        return out

    def free_seq(self, seq_id: int) -> None:
        _acheck(_lib.pkv_alloc_free_seq(self._h, int(seq_id)), "free_seq")

    def export(self, seq_ids, width: int):
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        tables = np.empty((len(ids), width), dtype=np.int32)
        lens = np.empty(len(ids), dtype=np.int32)
        _acheck(_lib.pkv_alloc_export(self._h, _addr(ids), len(ids), int(width), _addr(tables),
                                      _addr(lens)), "export")
        return tables, lens

    def stats(self):
        f, u, s, x = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64(), ctypes.c_double()
        _acheck(_lib.pkv_alloc_stats(self._h, ctypes.byref(f), ctypes.byref(u), ctypes.byref(s),
                                     ctypes.byref(x)), "stats")
        return f.value, u.value, s.value, x.value

    def free_blocks(self) -> list[int]:
        n = ctypes.c_int64()
        _acheck(_lib.pkv_alloc_free_list(self._h, None, 0, ctypes.byref(n)), "free_list")
        out = np.empty(n.value, dtype=np.int64)
        _acheck(_lib.pkv_alloc_free_list(self._h, out.ctypes.data if n.value else None, n.value,
                                         ctypes.byref(n)), "free_list")
        return out.tolist()

    def set_host_pool(self, num_host_blocks: int) -> None:
        _acheck(_lib.pkv_alloc_set_host_pool(self._h, int(num_host_blocks)), "set_host_pool")

    def swap_out(self, seq_id: int) -> None:
        _acheck(_lib.pkv_alloc_swap_out(self._h, int(seq_id)), "swap_out")

    def swap_in(self, seq_id: int) -> None:
        _acheck(_lib.pkv_alloc_swap_in(self._h, int(seq_id)), "swap_in")

    def take_swaps(self, direction: int):
        """Queued (gpu_block, host_slot) pairs of one direction; clears them."""
        n = ctypes.c_int64()
        _acheck(_lib.pkv_alloc_take_swaps(self._h, direction, None, None, 0, ctypes.byref(n)),
                "take_swaps")
        g = np.empty(n.value, np.int64)
        h = np.empty(n.value, np.int64)
        _acheck(_lib.pkv_alloc_take_swaps(self._h, direction, g.ctypes.data if n.value else None,
                                          h.ctypes.data if n.value else None, n.value,
                                          ctypes.byref(n)), "take_swaps")
        return g, h

    def take_copies(self):
        """Queued copy-on-write pairs (src, dst) as int64 arrays; clears the queue."""
        n = ctypes.c_int64()
        _acheck(_lib.pkv_alloc_take_copies(self._h, None, None, 0, ctypes.byref(n)), "take_copies")
        src = np.empty(n.value, np.int64)
        dst = np.empty(n.value, np.int64)
        _acheck(_lib.pkv_alloc_take_copies(self._h, src.ctypes.data if n.value else None,
                                           dst.ctypes.data if n.value else None, n.value,
                                           ctypes.byref(n)), "take_copies")
        return src, dst

    def prefix_groups(self, seq_ids):
        """(prefix_blocks [n], group_offsets [G + 1], group_seqs [members]) as int32
        arrays for paged_attention_decode_prefix; group_seqs index into seq_ids."""
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        n = len(ids)
        pb = np.zeros(n, np.int32)
        offs = np.zeros(n + 1, np.int32)
        members = np.zeros(max(n, 1), np.int32)
        g = ctypes.c_int32()
        _acheck(_lib.pkv_alloc_prefix_groups(self._h, ids.ctypes.data, n, pb.ctypes.data,
                                             offs.ctypes.data, members.ctypes.data,
                                             ctypes.byref(g)), "prefix_groups")
        return pb, offs[: g.value + 1].copy(), members[: offs[g.value]].copy()

    def refcount(self, block: int) -> int:
        out = ctypes.c_int32()
        _acheck(_lib.pkv_alloc_refcount(self._h, int(block), ctypes.byref(out)), "refcount")
        return out.value

    def seq_len(self, seq_id: int) -> int:
        out = ctypes.c_int64()
        _acheck(_lib.pkv_alloc_seq_len(self._h, int(seq_id), ctypes.byref(out)), "seq_len")
        return out.value

    def slot_of(self, seq_id: int, pos: int) -> int:
        out = ctypes.c_int64()
        _acheck(_lib.pkv_alloc_slot_of(self._h, int(seq_id), int(pos), ctypes.byref(out)), "slot_of")
        return out.value
