"""Shared helpers for the GPU parity tests: upload a seeded workload, run the
library's write + decode through the C ABI, and compare with the oracle."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from oracle.alloc_model import BlockManager
import workloads as wl

# Tolerance for bf16 attention outputs accumulated in fp32, against the fp64
# oracle: an element passes when |gpu - ref| <= ATOL + RTOL * |ref|.
ATOL = 1e-2
RTOL = 1e-2


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def host_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return wl.bf16_to_f32(bits).astype(np.float64)


def check_close(out_bits: np.ndarray, ref: np.ndarray, what: str = ""):
    got = bits_to_f64(out_bits)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    err = np.abs(got - ref)
    bad = err > ATOL + RTOL * np.abs(ref)
    big = np.abs(ref) >= 1e-3
    max_abs = float(err.max()) if err.size else 0.0
    max_rel = float((err[big] / np.abs(ref[big])).max()) if big.any() else 0.0
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {bad.size} elements out of tolerance; "
                           f"max abs {max_abs:.3g}, max rel {max_rel:.3g}")
    return max_abs, max_rel


class DeviceStep:
    """A workload resident on the GPU (pre-write caches, step inputs)."""

    def __init__(self, w: wl.Workload):
        self.w = w
        self.q = dev_bf16(w.q)
        self.k_new = dev_bf16(w.k_new)
        self.v_new = dev_bf16(w.v_new)
        self.kc = dev_bf16(w.k_cache)
        self.vc = dev_bf16(w.v_cache)
        self.tables = torch.from_numpy(w.block_tables).cuda()
        self.lens = torch.from_numpy(w.lens.astype(np.int32)).cuda()
        self.slots = torch.from_numpy(w.slot_mapping).cuda()
        self.err = torch.zeros(1, dtype=torch.int32, device="cuda")
        self.out = torch.empty_like(self.q)

    def write(self):
        from paged_kv_cache_459_b200 import pkv
        pkv.paged_kv_write(self.k_new, self.v_new, self.kc, self.vc, self.slots, err=self.err)

    def decode(self, variant=0, partition_tokens=512, tables=None, lens=None):
        from paged_kv_cache_459_b200 import pkv
        pkv.paged_attention_decode(self.out, self.q, self.kc, self.vc,
                                   self.tables if tables is None else tables,
                                   self.lens if lens is None else lens,
                                   self.w.cfg["scale"], self.w.cfg["num_kv_heads"],
                                   variant=variant, partition_tokens=partition_tokens, err=self.err)
        torch.cuda.synchronize()
        return host_bits(self.out)

    def err_word(self) -> int:
        torch.cuda.synchronize()
        return int(self.err.item())


def oracle_after_write(w: wl.Workload):
    """The oracle's post-write caches and its fp64 decode of the step."""
    kc, vc = oracle.kv_write(w.k_cache, w.v_cache, w.k_new, w.v_new, w.slot_mapping)
    ref = oracle.paged_decode(w.q, kc, vc, w.block_tables, w.lens, w.cfg["scale"])
    return kc, vc, ref


def build(name, seed, **kw) -> wl.Workload:
    return wl.build(name, seed, BlockManager, **kw)
