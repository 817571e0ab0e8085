"""Seeded synthetic inputs for paged decode attention.

This module only draws random numbers and lays them out: sequence lengths,
the order of the free-block list, bf16 Q/K/V values and NaN poison.  It holds
no attention arithmetic and no allocation policy.  Block tables and slots come
from an allocator object that the caller passes in (the library's C++ block
allocator, or the reference model under ``oracle/``), which is how both the
CUDA path and the oracle are fed the same inputs without sharing code.  It
sits outside both the library package and ``oracle/`` and imports neither.

Workloads (the shapes come from the decode configurations this library is
measured on):

=========  =====  ======  ===  ===========================================
name       B      Hq/Hkv  d    lengths and pool
=========  =====  ======  ===  ===========================================
tiny       4      4/4     64   {1, 17, 33, 100}; 64-block pool, scale 1/8
llama      64     32/32   128  U[128, 2048]; pool 1.1x need
qwen       256    28/4    128  U[512, 4096]; pool 1.1x need (fragmented)
prefix     128    32/32   128  2000-token shared prefix + U[16, 512] suffix
long       8      32/8    128  32768 each; 20000-block pool
=========  =====  ======  ===  ===========================================

Values are bf16 = round-to-nearest-even of N(0, 1) float32 draws from PCG64
generators (one per 4M-element chunk, keyed by seed, stream and chunk).
Every block starts with random values; blocks that no table uses, the unused
tail slots of each sequence's last block and the slot of the new token are
then set to bf16 NaN so that a stray read shows up in the output.
"""
from __future__ import annotations

import math
import os
from dataclasses import dataclass, field

import numpy as np

BLOCK_TOKENS = 16
BF16_NAN = np.uint16(0x7FC0)

CONFIGS: dict[str, dict] = {
    "tiny": dict(batch=4, num_heads=4, num_kv_heads=4, head_dim=64,
                 lens=(1, 17, 33, 100), num_blocks=64, scale=1.0 / 8.0),
    "llama": dict(batch=64, num_heads=32, num_kv_heads=32, head_dim=128,
                  len_lo=128, len_hi=2048, pool_factor=1.1),
    "qwen": dict(batch=256, num_heads=28, num_kv_heads=4, head_dim=128,
                 len_lo=512, len_hi=4096, pool_factor=1.1),
    "prefix": dict(batch=128, num_heads=32, num_kv_heads=32, head_dim=128,
                   prefix_len=2000, suffix_lo=16, suffix_hi=512, pool_factor=1.1),
    "long": dict(batch=8, num_heads=32, num_kv_heads=8, head_dim=128,
                 len_fixed=32768, num_blocks=20000, partition_tokens=512),
}


def config(name: str, **overrides) -> dict:
    cfg = dict(CONFIGS[name])
    cfg.update(overrides)
    cfg["name"] = name
    if "scale" not in cfg:
        cfg["scale"] = 1.0 / math.sqrt(cfg["head_dim"])
    return cfg


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


_CHUNK = 1 << 22


def _normal_chunk(args):
    seed, stream, c, n = args
    gen = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, stream, c])))
    f = gen.standard_normal(n, dtype=np.float32)
    u = f.view(np.uint32)
    # round to nearest even on the upper 16 bits; the draws are finite
    u += np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return (u >> np.uint32(16)).astype(np.uint16)


def bf16_normal(shape, seed: int, stream: int) -> np.ndarray:
    """bf16 bit patterns (uint16) of round-to-nearest-even N(0,1) float32 draws.

    Element i of stream ``stream`` comes from chunk i // 2^22, drawn by its own
    PCG64 seeded with SeedSequence([seed, stream, chunk]); chunks are drawn in
    parallel threads, so the values do not depend on the thread count."""
    n = int(np.prod(shape))
    jobs = [(int(seed), int(stream), c, min(_CHUNK, n - c * _CHUNK))
            for c in range(-(-n // _CHUNK))]
    if len(jobs) <= 1:
        parts = [_normal_chunk(j) for j in jobs]
    else:
        from concurrent.futures import ThreadPoolExecutor
        with ThreadPoolExecutor(max_workers=min(len(jobs), os.cpu_count() or 1)) as ex:
            parts = list(ex.map(_normal_chunk, jobs))
    out = np.concatenate(parts) if parts else np.empty(0, np.uint16)
    return out.reshape(shape)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


def draw_lens(cfg: dict, gen: np.random.Generator) -> np.ndarray:
    """Per-sequence context lengths, counting the token decoded this step."""
    b = cfg["batch"]
    if "lens" in cfg:
        lens = np.array(cfg["lens"], dtype=np.int64)
        assert len(lens) == b
        return lens
    if "len_fixed" in cfg:
        return np.full(b, cfg["len_fixed"], dtype=np.int64)
    if "prefix_len" in cfg:
        suf = gen.integers(cfg["suffix_lo"], cfg["suffix_hi"], size=b, endpoint=True)
        return cfg["prefix_len"] + suf.astype(np.int64)
    return gen.integers(cfg["len_lo"], cfg["len_hi"], size=b, endpoint=True).astype(np.int64)


def _shares_prefix(cfg: dict, s: int) -> bool:
    every = cfg.get("unshared_every", 0)
    return "prefix_len" in cfg and not (every and s % every == every - 1)


def pool_blocks(cfg: dict, lens: np.ndarray) -> int:
    if "num_blocks" in cfg:
        return int(cfg["num_blocks"])
    nb = lambda n: -(-int(n) // BLOCK_TOKENS)  # noqa: E731  (blocks to hold n tokens)
    if "prefix_len" in cfg:
        pl = cfg["prefix_len"]
        need = nb(pl) * cfg.get("prefix_groups", 1) + sum(
            nb(int(l) - pl) if _shares_prefix(cfg, s) else nb(int(l)) for s, l in enumerate(lens))
    else:
        need = sum(nb(int(l)) for l in lens)
    return int(math.ceil(cfg["pool_factor"] * need))


@dataclass
class Workload:
    cfg: dict
    seed: int
    lens: np.ndarray            # int32 [B]   tokens per sequence incl. the new one
    block_tables: np.ndarray    # int32 [B, W]; -1 beyond each sequence's blocks
    slot_mapping: np.ndarray    # int64 [B]   slot of the new token
    num_blocks: int
    q: np.ndarray               # uint16 bf16 bits [B, Hq, d]
    k_new: np.ndarray           # uint16 [B, Hkv, d]
    v_new: np.ndarray           # uint16 [B, Hkv, d]
    k_cache: np.ndarray | None  # uint16 [NB, Hkv, 16, d]  (pre-write image)
    v_cache: np.ndarray | None
    free_blocks: np.ndarray = field(default_factory=lambda: np.zeros(0, np.int64))
    alloc: object = None

    @property
    def width(self) -> int:
        return int(self.block_tables.shape[1])


def build(name: str, seed: int, alloc_factory, *, batch: int | None = None,
          with_cache: bool = True, poison: bool = True, width: int | None = None,
          **overrides) -> Workload:
    """Draw one decode step of workload ``name``.

    ``alloc_factory(num_blocks, free_order)`` returns an allocator with
    ``add_seq``, ``fork``, ``append_token``, ``free_seq``, ``export`` and
    ``free_blocks``.  The recipe: every sequence is prefilled with len-1
    tokens, then one token is appended, whose slot is the step's
    ``slot_mapping`` entry.  In the ``prefix`` workload a 2000-token prefix is
    prefilled once, forked into every sequence and then released by its owner,
    so its blocks are shared by all ``batch`` tables (``prefix_groups`` > 1:
    that many prefixes, sequence s joining group s % prefix_groups;
    ``unshared_every`` = n: every n-th sequence holds no shared prefix).
    """
    cfg = config(name, **overrides)
    if batch is not None:
        cfg["batch"] = batch
        if "lens" in cfg:
            cfg["lens"] = tuple(cfg["lens"][:batch])
    gen = rng(seed)
    lens = draw_lens(cfg, gen)
    nblocks = pool_blocks(cfg, lens)
    free_order = gen.permutation(nblocks).astype(np.int64)
    alloc = alloc_factory(nblocks, free_order)
    b = cfg["batch"]
    seq_ids = list(range(b))
    if "prefix_len" in cfg:
        # owners of the shared prefixes get ids outside the batch
        owners = [b + g for g in range(cfg.get("prefix_groups", 1))]
        for o in owners:
            alloc.add_seq(o, cfg["prefix_len"])
        for s in seq_ids:
            if _shares_prefix(cfg, s):
                alloc.fork(owners[s % len(owners)], s)
                for _ in range(int(lens[s]) - 1 - cfg["prefix_len"]):
                    alloc.append_token(s)
            else:
                alloc.add_seq(s, int(lens[s]) - 1)
        for o in owners:
            alloc.free_seq(o)
    else:
        for s in seq_ids:
            alloc.add_seq(s, int(lens[s]) - 1)
    slots = np.array([alloc.append_token(s) for s in seq_ids], dtype=np.int64)
    w = width if width is not None else max(1, max(-(-int(l) // BLOCK_TOKENS) for l in lens))
    tables, out_lens = alloc.export(seq_ids, w)
    assert np.array_equal(out_lens.astype(np.int64), lens)
    hq, hkv, d = cfg["num_heads"], cfg["num_kv_heads"], cfg["head_dim"]
    q = bf16_normal((b, hq, d), seed, 1)
    k_new = bf16_normal((b, hkv, d), seed, 2)
    v_new = bf16_normal((b, hkv, d), seed, 3)
    free = np.asarray(alloc.free_blocks(), dtype=np.int64)
    kc = vc = None
    if with_cache:
        kc = bf16_normal((nblocks, hkv, BLOCK_TOKENS, d), seed, 4)
        vc = bf16_normal((nblocks, hkv, BLOCK_TOKENS, d), seed, 5)
        if poison:
            poison_cache(kc, vc, free, tables, out_lens, slots)
    return Workload(cfg=cfg, seed=seed, lens=out_lens.astype(np.int32), block_tables=tables,
                    slot_mapping=slots, num_blocks=nblocks, q=q, k_new=k_new, v_new=v_new,
                    k_cache=kc, v_cache=vc, free_blocks=free, alloc=alloc)


def poison_cache(kc, vc, free_blocks, tables, lens, new_slots) -> None:
    """NaN in free blocks, in slots past each sequence's end and in the slot
    the step's write must fill.  Cache layout: [block][kv head][16][d]."""
    if len(free_blocks):
        kc[free_blocks] = BF16_NAN
        vc[free_blocks] = BF16_NAN
    for b, n in enumerate(np.asarray(lens)):
        n = int(n)
        if n % BLOCK_TOKENS:
            blk = int(tables[b, (n - 1) // BLOCK_TOKENS])
            kc[blk, :, n % BLOCK_TOKENS:, :] = BF16_NAN
            vc[blk, :, n % BLOCK_TOKENS:, :] = BF16_NAN
    for s in np.asarray(new_slots):
        s = int(s)
        if s >= 0:
            kc[s // BLOCK_TOKENS, :, s % BLOCK_TOKENS, :] = BF16_NAN
            vc[s // BLOCK_TOKENS, :, s % BLOCK_TOKENS, :] = BF16_NAN
