"""fp64 CPU oracle for paged decode attention and the paged KV-cache write.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this package.  It shares no code with
the CUDA library package and never imports it; the only module both sides use
is the seeded input generator (``workloads.py`` at the repository root), which
holds no attention arithmetic and imports neither side.

* ``paged_decode``          -- softmax(scale * q K^T) V per (sequence, query head),
                               K and V gathered through the block table (C, fp64).
* ``paged_decode_partitioned`` -- the same in independent token partitions
                               combined by log-sum-exp (C, fp64).
* ``paged_prefill``         -- causal attention of new (prompt) tokens: each row
                               is the decode definition at its own position.
* ``kv_write``              -- the new token's K/V copied into its slot (C).
* ``copy_blocks``           -- copy-on-write copies of whole blocks (C).
* ``swap_blocks``           -- blocks moved to / from host swap space (C).
* ``alloc_model.BlockManager`` -- the block allocator's reference model (Python).

Pins (all CPU tests): the pages' worked block-table, waste and sharing
examples; closed forms (len 1, equal keys, two keys, one dominant key); brute
force against torch's fp64 scaled_dot_product_attention on un-paged K/V;
invariance under physical-block relabelling; the partition identity.
No function here is left unpinned.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        path = _build.build()
        l = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i32, i64, f64 = ctypes.c_int, ctypes.c_int64, ctypes.c_double
        l.oracle_kv_write.argtypes = [P, P, P, P, P, i64, i32, i32, i64]
        l.oracle_kv_write.restype = i32
        l.oracle_paged_decode.argtypes = [P, P, P, P, P, i32, P, i32, i32, i32, i32, i64, f64, i32]
        l.oracle_paged_decode.restype = i32
        l.oracle_paged_decode_partitioned.argtypes = [P, P, P, P, P, i32, P, i32, i32, i32, i32,
                                                      i64, f64, i32]
        l.oracle_paged_decode_partitioned.restype = i32
        l.oracle_block_tokens.restype = i32
        l.oracle_copy_blocks.argtypes = [P, P, P, P, i64, i32, i32, i64]
        l.oracle_copy_blocks.restype = i32
        l.oracle_swap_blocks.argtypes = [P, P, P, P, P, P, i64, i32, i32, i32, i64, i64]
        l.oracle_swap_blocks.restype = i32
        _lib = l
    return _lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16, "bf16 inputs are passed as uint16 bit patterns"
    return a


def block_tokens() -> int:
    return int(lib().oracle_block_tokens())


def kv_write(k_cache, v_cache, k, v, slot_mapping):
    """Return copies of the caches after writing k/v [T, Hkv, d] at the slots."""
    kc, vc = np.array(_u16(k_cache), copy=True), np.array(_u16(v_cache), copy=True)
    k, v = _u16(k), _u16(v)
    slots = np.ascontiguousarray(slot_mapping, dtype=np.int64)
    nb, hkv, bt, d = kc.shape
    assert bt == block_tokens() and k.shape == (len(slots), hkv, d) and v.shape == k.shape
    valid = slots[slots >= 0]
    if len(np.unique(valid)) != len(valid):
        raise ValueError("duplicate slots in one write")
    rc = lib().oracle_kv_write(_ptr(kc), _ptr(vc), _ptr(k), _ptr(v), _ptr(slots), len(slots),
                               hkv, d, nb)
    if rc:
        raise ValueError("slot outside the pool")
    return kc, vc


def copy_blocks(k_cache, v_cache, src, dst):
    """Copies of the caches after copying block src[i] to dst[i] for every i."""
    kc, vc = np.array(_u16(k_cache), copy=True), np.array(_u16(v_cache), copy=True)
    s = np.ascontiguousarray(src, dtype=np.int64)
    d = np.ascontiguousarray(dst, dtype=np.int64)
    nb, hkv, bt, hd = kc.shape
    if lib().oracle_copy_blocks(_ptr(kc), _ptr(vc), _ptr(s), _ptr(d), len(s), hkv, hd, nb):
        raise ValueError("block id outside the pool")
    return kc, vc


def swap_blocks(k_cache, v_cache, host_k, host_v, gpu, host, direction):
    """(k_cache, v_cache, host_k, host_v) after moving blocks between the cache
    and the host swap space (direction 0: out, 1: in); all copies."""
    kc, vc = np.array(_u16(k_cache), copy=True), np.array(_u16(v_cache), copy=True)
    hk, hv = np.array(_u16(host_k), copy=True), np.array(_u16(host_v), copy=True)
    g = np.ascontiguousarray(gpu, dtype=np.int64)
    h = np.ascontiguousarray(host, dtype=np.int64)
    nb, hkv, bt, d = kc.shape
    if lib().oracle_swap_blocks(_ptr(kc), _ptr(vc), _ptr(hk), _ptr(hv), _ptr(g), _ptr(h), len(g),
                                int(direction), hkv, d, nb, hk.shape[0]):
        raise ValueError("block id outside the pool or the swap space")
    return kc, vc, hk, hv


def paged_decode(q, k_cache, v_cache, block_tables, seq_lens, scale, nthreads: int = 0):
    """fp64 attention output [B, Hq, d]."""
    q, kc, vc = _u16(q), _u16(k_cache), _u16(v_cache)
    tables = np.ascontiguousarray(block_tables, dtype=np.int32)
    lens = np.ascontiguousarray(seq_lens, dtype=np.int32)
    b, hq, d = q.shape
    nb, hkv = kc.shape[0], kc.shape[1]
    out = np.zeros((b, hq, d), dtype=np.float64)
    rc = lib().oracle_paged_decode(_ptr(out), _ptr(q), _ptr(kc), _ptr(vc), _ptr(tables),
                                   tables.shape[1], _ptr(lens), b, hq, hkv, d, nb, float(scale),
                                   int(nthreads))
    if rc:
        raise ValueError(f"oracle_paged_decode failed ({rc})")
    return out


def paged_prefill(q, k_cache, v_cache, block_tables, seq_lens, query_start, scale):
    """Causal prefill: row r of sequence b (query_start[b] <= r < query_start[b+1])
    is the token at position p = seq_lens[b] - n_b + (r - query_start[b]) and
    attends to positions [0, p] -- the decode definition with length p + 1."""
    qs = np.asarray(query_start, dtype=np.int64)
    lens = np.asarray(seq_lens, dtype=np.int64)
    tables = np.asarray(block_tables, dtype=np.int32)
    rows_seq = np.repeat(np.arange(len(lens)), np.diff(qs))
    first = lens[rows_seq] - np.diff(qs)[rows_seq]
    pos = first + (np.arange(qs[-1]) - qs[rows_seq])
    return paged_decode(q, k_cache, v_cache, tables[rows_seq], (pos + 1).astype(np.int32), scale)


def paged_decode_partitioned(q, k_cache, v_cache, block_tables, seq_lens, scale, partition_tokens):
    q, kc, vc = _u16(q), _u16(k_cache), _u16(v_cache)
    tables = np.ascontiguousarray(block_tables, dtype=np.int32)
    lens = np.ascontiguousarray(seq_lens, dtype=np.int32)
    b, hq, d = q.shape
    nb, hkv = kc.shape[0], kc.shape[1]
    out = np.zeros((b, hq, d), dtype=np.float64)
    rc = lib().oracle_paged_decode_partitioned(_ptr(out), _ptr(q), _ptr(kc), _ptr(vc),
                                               _ptr(tables), tables.shape[1], _ptr(lens), b, hq,
                                               hkv, d, nb, float(scale), int(partition_tokens))
    if rc:
        raise ValueError(f"oracle_paged_decode_partitioned failed ({rc})")
    return out


def threads_available() -> int:
    return len(os.sched_getaffinity(0))
