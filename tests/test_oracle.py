"""Pins for the fp64 oracle: the pages' worked examples, closed forms, brute
force against torch's fp64 attention on un-paged K/V, and invariants.  None of
them re-types the oracle's own formula; each is chosen so that a plausible
slip in it (a swapped block/offset index, a dropped scale, a wrong GQA group,
an off-by-one length) fails at least one of them -- ``test_planted_mistakes``
checks that directly."""
import json
import os
import shutil
import subprocess

import numpy as np
import pytest
import scipy.special
import torch
import torch.nn.functional as F

import oracle
from oracle.alloc_model import BlockManager
import workloads as wl
from relabel import permute_pool

BT = 16


def rb(shape, gen):
    """Seeded bf16 N(0,1) bits, the seed drawn from `gen`."""
    return wl.bf16_normal(shape, int(gen.integers(1 << 31)), 0)


def f32(bits):
    return wl.bf16_to_f32(np.asarray(bits, dtype=np.uint16)).astype(np.float64)


def page_sequences(ks, vs, num_blocks, seed, lib=None):
    """Write per-sequence contiguous K/V ([len, Hkv, d] bf16 bits) into a
    paged pool token by token, with slots handed out by the allocator model
    and the oracle's write.  Returns (k_cache, v_cache, tables, lens)."""
    gen = wl.rng(seed)
    hkv, d = ks[0].shape[1], ks[0].shape[2]
    bm = BlockManager(num_blocks, gen.permutation(num_blocks))
    kc = rb((num_blocks, hkv, BT, d), gen)
    vc = rb((num_blocks, hkv, BT, d), gen)
    slots, krows, vrows = [], [], []
    for s, (k, v) in enumerate(zip(ks, vs)):
        bm.add_seq(s, 0)
        for p in range(k.shape[0]):
            slots.append(bm.append_token(s))
            krows.append(k[p])
            vrows.append(v[p])
    if slots:
        kc, vc = oracle.kv_write(kc, vc, np.stack(krows), np.stack(vrows), np.array(slots))
    width = max(1, max(-(-k.shape[0] // BT) for k in ks))
    tables, lens = bm.export(list(range(len(ks))), width)
    return kc, vc, tables, lens


def sdpa_reference(q_bits, ks, vs, scale):
    """torch fp64 scaled_dot_product_attention on un-paged K/V, per sequence."""
    out = []
    for b, (k, v) in enumerate(zip(ks, vs)):
        qt = torch.from_numpy(f32(q_bits[b]))[None, :, None, :]           # [1, Hq, 1, d]
        kt = torch.from_numpy(f32(k)).permute(1, 0, 2)[None]               # [1, Hkv, L, d]
        vt = torch.from_numpy(f32(v)).permute(1, 0, 2)[None]
        o = F.scaled_dot_product_attention(qt, kt, vt, scale=scale, enable_gqa=True)
        out.append(o[0, :, 0, :].numpy())
    return np.stack(out)


def random_case(seed, lens, hq, hkv, d):
    gen = wl.rng(seed)
    ks = [rb((n, hkv, d), gen) for n in lens]
    vs = [rb((n, hkv, d), gen) for n in lens]
    q = rb((len(lens), hq, d), gen)
    return q, ks, vs


# --------------------------------------------------------------- worked examples
def test_block_table_example(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "block_table_example.json")))
    table = g["printed"]["request_A_block_table"]
    order = [table["0"], table["1"], table["2"]]
    order += [b for b in range(64) if b not in order]
    bm = BlockManager(64, order)
    bm.add_seq("A", 48)
    assert bm.tables["A"] == [table["0"], table["1"], table["2"]]
    for tok, (blk, off) in g["expected_physical_block_and_offset_by_token"].items():
        slot = bm.slot_of("A", int(tok) - 1)
        assert (slot // BT, slot % BT) == (blk, off)
        assert slot == g["expected_slot_by_token"][tok]
    # the same slots through the write oracle: token t lands at [block][h][offset]
    d, hkv = 8, 2
    kc = np.zeros((64, hkv, BT, d), np.uint16)
    toks = sorted(int(t) for t in g["expected_slot_by_token"])
    k = np.array([[[t] * d] * hkv for t in toks], np.uint16)
    slots = np.array([g["expected_slot_by_token"][str(t)] for t in toks])
    kc2, _ = oracle.kv_write(kc, kc, k, k, slots)
    for t in toks:
        blk, off = g["expected_physical_block_and_offset_by_token"][str(t)]
        assert (kc2[blk, :, off, :] == t).all()
    assert np.count_nonzero(kc2) == len(toks) * hkv * d


def test_waste_examples(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "waste_examples.json")))
    for c in g["cases"]:
        assert g["reserved_tokens"] - c["used"] == c["contiguous_wasted"]
        if "contiguous_waste_pct" in c:
            assert round(100 * c["contiguous_wasted"] / g["reserved_tokens"]) == c["contiguous_waste_pct"]
        bm = BlockManager(256)
        bm.add_seq(0, c["used"])
        free, used, shared, util = bm.stats()
        assert used == c["paged_blocks"] == len(bm.tables[0])
        assert BT * used - c["used"] == c["paged_wasted"]
        assert c["paged_wasted"] < BT  # at most one partly filled block
        assert util == pytest.approx(c["used"] / (BT * used))


def test_sharing_example(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "sharing_example.json")))
    bm = BlockManager(16, list(range(1, 16)) + [0])
    bm.add_seq("A", 64)
    bm.fork("A", "B", 48)
    for _ in range(16):
        bm.append_token("B")
    bm.fork("A", "C", 32)
    for _ in range(32):
        bm.append_token("C")
    for name, table in g["printed"]["tables"].items():
        assert bm.tables[name] == table
    for blk, rc in g["expected_refcounts"].items():
        assert bm.refcount(int(blk)) == rc
    assert bm.stats()[2] == 3  # blocks 1, 2, 3 are shared
    bm.free_seq("A")
    for blk, rc in g["expected_after_freeing_A"]["refcounts"].items():
        assert bm.refcount(int(blk)) == rc
    assert bm.free_blocks()[-len(g["expected_after_freeing_A"]["freed"]):] == \
        g["expected_after_freeing_A"]["freed"]


def test_prefix_example(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "prefix_example.json")))
    bm = BlockManager(512)
    bm.add_seq("sys", g["prefix_tokens"])
    assert len(bm.tables["sys"]) == g["expected_prefix_blocks"]
    assert g["prefix_tokens"] % BT == 0 and g["expected_partial_blocks"] == 0
    for c in range(4):
        bm.fork("sys", c)
        bm.append_token(c)  # the prefix's last block is full: a private block opens
        assert bm.tables[c][:125] == bm.tables["sys"] and len(bm.tables[c]) == 126
    assert all(bm.refcount(b) == 5 for b in bm.tables["sys"])


def test_lifecycle_steps():
    """Steps 一 to 四 of the request lifecycle."""
    bm = BlockManager(8, [3, 1, 4, 0, 5, 2, 7, 6])
    bm.add_seq("r", 0)                                # 一: empty table, nothing reserved
    assert bm.tables["r"] == [] and bm.stats()[1] == 0
    slots = [bm.append_token("r") for _ in range(16)]  # 二/三: one block until it fills
    assert bm.tables["r"] == [3] and slots == list(range(48, 64))
    assert bm.append_token("r") == 16                 # full -> a new block (id 1)
    assert bm.tables["r"] == [3, 1]
    bm.free_seq("r")                                  # 四: every block back to the pool
    assert bm.stats()[1] == 0 and bm.free_blocks()[-2:] == [3, 1]
    bm.add_seq("s", 40)                               # freed blocks serve anyone
    assert len(bm.tables["s"]) == 3


def test_allocator_errors_leave_state_unchanged():
    bm = BlockManager(4)
    bm.add_seq(0, 40)
    before = (list(bm.free), list(bm.ref), {k: list(v) for k, v in bm.tables.items()}, dict(bm.lens))
    for call in (lambda: bm.add_seq(1, 33), lambda: bm.add_seq(0, 1), lambda: bm.fork(0, 0),
                 lambda: bm.fork(9, 1), lambda: bm.free_seq(7), lambda: bm.fork(0, 1, 41)):
        with pytest.raises(Exception):
            call()
        assert (list(bm.free), list(bm.ref), {k: list(v) for k, v in bm.tables.items()},
                dict(bm.lens)) == before
    bm.fork(0, 1)  # shares the partly filled third block
    shared = bm.tables[0][2]
    slot = bm.append_token(1)  # copy-on-write: a private copy of the shared block
    assert bm.tables[1][:2] == bm.tables[0][:2] and bm.tables[1][2] != shared
    assert slot == bm.tables[1][2] * 16 + 8 and bm.refcount(shared) == 1
    assert [tuple(x) for x in zip(*bm.take_copies())] == [(shared, bm.tables[1][2])]
    assert bm.take_copies()[0].size == 0
    with pytest.raises(Exception) as e:
        bm.add_seq(3, 1)
    assert e.value.kind == "oom"


# ------------------------------------------------------------------ brute force
@pytest.mark.parametrize("d,hq,hkv,lens", [
    (64, 4, 4, [1, 17, 33, 100]),
    (128, 8, 2, [16, 15, 47, 64]),
    (64, 28, 4, [5, 130]),
    (32, 3, 1, [2, 31, 32, 33]),
    (128, 32, 8, [257]),
])
def test_oracle_matches_library_attention(d, hq, hkv, lens):
    q, ks, vs = random_case(7 + d + hq, lens, hq, hkv, d)
    kc, vc, tables, lens_ = page_sequences(ks, vs, 64, seed=11)
    scale = 1.0 / np.sqrt(d)
    got = oracle.paged_decode(q, kc, vc, tables, lens_, scale)
    want = sdpa_reference(q, ks, vs, scale)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_empty_sequence_gives_zero():
    q, ks, vs = random_case(3, [0, 5], 2, 2, 64)
    kc, vc, tables, lens = page_sequences(ks, vs, 8, seed=1)
    out = oracle.paged_decode(q, kc, vc, tables, lens, 0.125)
    assert (out[0] == 0).all() and np.isfinite(out).all()


# ------------------------------------------------------------------ closed forms
def test_len_one_returns_v_exactly():
    q, ks, vs = random_case(5, [1, 1, 1], 4, 2, 64)
    kc, vc, tables, lens = page_sequences(ks, vs, 8, seed=2)
    out = oracle.paged_decode(q, kc, vc, tables, lens, 0.125)
    for b in range(3):
        for h in range(4):
            assert np.array_equal(out[b, h], f32(vs[b][0, h // 2]))


def test_equal_keys_or_zero_scale_average_v():
    q, ks, vs = random_case(6, [37], 4, 4, 64)
    ks[0][:] = ks[0][0]  # all keys equal
    kc, vc, tables, lens = page_sequences(ks, vs, 8, seed=3)
    mean_v = f32(vs[0]).mean(axis=0)  # [Hkv, d]
    out = oracle.paged_decode(q, kc, vc, tables, lens, 0.125)
    np.testing.assert_allclose(out[0], mean_v, rtol=0, atol=1e-12)
    q2, ks2, vs2 = random_case(8, [50], 4, 4, 64)
    kc, vc, tables, lens = page_sequences(ks2, vs2, 8, seed=4)
    out = oracle.paged_decode(q2, kc, vc, tables, lens, 0.0)
    np.testing.assert_allclose(out[0], f32(vs2[0]).mean(axis=0), rtol=0, atol=1e-12)


def test_two_keys_logistic_weights():
    q, ks, vs = random_case(9, [2], 2, 1, 64)
    kc, vc, tables, lens = page_sequences(ks, vs, 8, seed=5)
    scale = 0.3
    out = oracle.paged_decode(q, kc, vc, tables, lens, scale)
    k, v = f32(ks[0])[:, 0], f32(vs[0])[:, 0]
    for h in range(2):
        qh = f32(q[0, h])
        w0 = scipy.special.expit(scale * (np.dot(qh, k[0]) - np.dot(qh, k[1])))
        np.testing.assert_allclose(out[0, h], w0 * v[0] + (1 - w0) * v[1], rtol=0, atol=1e-12)


def test_dominant_key_is_one_hot():
    d = 64
    gen = wl.rng(10)
    q = rb((1, 1, d), gen)
    k = rb((40, 1, d), gen)
    v = rb((40, 1, d), gen)
    # key 23 = 64 * q (exact in bf16: power-of-two multiple), so its score dominates by ~1e3
    k[23, 0] = (wl.bf16_to_f32(q[0, 0]) * 64).astype(np.float32).view(np.uint32) >> 16
    kc, vc, tables, lens = page_sequences([k], [v], 8, seed=6)
    out = oracle.paged_decode(q, kc, vc, tables, lens, 1.0)
    np.testing.assert_allclose(out[0, 0], f32(v[23, 0]), rtol=0, atol=1e-12)
    assert np.isfinite(out).all()  # exp(s - max) never overflows


# ------------------------------------------------------------------- invariants
def test_block_relabelling_invariance_is_bit_exact():
    w = wl.build("tiny", 0, BlockManager)
    kc, vc = oracle.kv_write(w.k_cache, w.v_cache, w.k_new, w.v_new, w.slot_mapping)
    base = oracle.paged_decode(w.q, kc, vc, w.block_tables, w.lens, w.cfg["scale"])
    for seed in range(3):
        perm = wl.rng(100 + seed).permutation(w.num_blocks)
        t2, _, kc2, vc2 = permute_pool(perm, w.block_tables, w.slot_mapping, kc, vc)
        out = oracle.paged_decode(w.q, kc2, vc2, t2, w.lens, w.cfg["scale"])
        assert np.array_equal(out, base)


def test_shared_prefix_equals_private_copy():
    """Sequences whose tables point at shared prefix blocks attend exactly as
    if each held a private copy of the prefix."""
    w = wl.build("prefix", 1, BlockManager, batch=4, prefix_len=64, suffix_lo=3, suffix_hi=40)
    kc, vc = oracle.kv_write(w.k_cache, w.v_cache, w.k_new, w.v_new, w.slot_mapping)
    shared = w.block_tables[:, :4]
    assert (shared == shared[0]).all() and all(w.alloc.refcount(int(b)) == 4 for b in shared[0])
    out = oracle.paged_decode(w.q, kc, vc, w.block_tables, w.lens, w.cfg["scale"])
    # give sequence b its own copy of the 4 prefix blocks in fresh pool slots
    nb = w.num_blocks
    kc2 = np.concatenate([kc] + [kc[shared[0]]] * 4)
    vc2 = np.concatenate([vc] + [vc[shared[0]]] * 4)
    t2 = w.block_tables.copy()
    for b in range(4):
        t2[b, :4] = nb + 4 * b + np.arange(4)
    out2 = oracle.paged_decode(w.q, kc2, vc2, t2, w.lens, w.cfg["scale"])
    assert np.array_equal(out, out2)


def test_poisoned_free_and_tail_slots_never_reach_output():
    for name, kw in (("tiny", {}), ("qwen", dict(batch=6, len_lo=1, len_hi=70))):
        w = wl.build(name, 2, BlockManager, **kw)
        kc, vc = oracle.kv_write(w.k_cache, w.v_cache, w.k_new, w.v_new, w.slot_mapping)
        assert np.isnan(f32(kc)).any()  # the poison is there
        out = oracle.paged_decode(w.q, kc, vc, w.block_tables, w.lens, w.cfg["scale"])
        assert np.isfinite(out).all()


def test_waste_bound_on_workloads():
    for name, kw in (("llama", dict(batch=16)), ("qwen", dict(batch=16)),
                     ("prefix", dict(batch=8))):
        w = wl.build(name, 3, BlockManager, with_cache=False, **kw)
        for b, n in enumerate(w.lens):
            nblk = int((w.block_tables[b] >= 0).sum())
            assert 0 <= BT * nblk - int(n) < BT


def test_partitioned_merge_equals_single_pass():
    for lens, part in (([1, 17, 33, 100], 16), ([700, 513, 512, 1], 512), ([1000], 48)):
        q, ks, vs = random_case(12, lens, 8, 2, 64)
        kc, vc, tables, lens_ = page_sequences(ks, vs, 128, seed=7)
        a = oracle.paged_decode(q, kc, vc, tables, lens_, 0.125)
        b = oracle.paged_decode_partitioned(q, kc, vc, tables, lens_, 0.125, part)
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


def test_write_skips_negative_slots_and_rejects_bad_ones():
    gen = wl.rng(4)
    kc = rb((4, 2, BT, 8), gen)
    k = rb((3, 2, 8), gen)
    k2, _ = oracle.kv_write(kc, kc, k, k, np.array([-1, 5, -7]))
    diff = np.argwhere((k2 != kc).any(axis=-1))
    assert set(map(tuple, diff[:, [0, 2]])) <= {(0, 5)}
    assert np.array_equal(k2[0, :, 5], k[1])
    with pytest.raises(ValueError):
        oracle.kv_write(kc, kc, k, k, np.array([0, 64, 1]))
    with pytest.raises(ValueError):
        oracle.kv_write(kc, kc, k, k, np.array([3, 3, 1]))


def test_oracle_threads_do_not_change_result():
    w = wl.build("qwen", 5, BlockManager, batch=5, len_lo=20, len_hi=200, poison=False)
    a = oracle.paged_decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.lens, w.cfg["scale"], 1)
    b = oracle.paged_decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.lens, w.cfg["scale"], 4)
    assert np.array_equal(a, b)


# ------------------------------------------------------------ planted mistakes
MUTATIONS = {
    "block and offset swapped": ("table_row[p / ORACLE_BLOCK_TOKENS]", "table_row[p % ORACLE_BLOCK_TOKENS]"),
    "scale dropped": ("s[p] = scale * acc;", "s[p] = acc;"),
    "query heads grouped modulo": ("for (int h = kvh * group; h < (kvh + 1) * group; ++h)",
                                   "for (int h = kvh; h < num_heads; h += num_kv_heads)"),
    "last token dropped": ("for (int p = 0; p < len; ++p) {\n        double acc",
                           "for (int p = 0; p < len - 1; ++p) {\n        double acc"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistakes_are_caught(name, tmp_path):
    """Compile a copy of the oracle with one plausible mistake; at least one
    pin must reject it."""
    if shutil.which("gcc") is None:
        pytest.skip("gcc missing")
    src = open(os.path.join(os.path.dirname(oracle.__file__), "oracle.c")).read()
    old, new = MUTATIONS[name]
    assert old in src, name
    (tmp_path / "m.c").write_text(src.replace(old, new))
    so = tmp_path / "m.so"
    subprocess.run(["gcc", "-O1", "-shared", "-fPIC", "-fopenmp", "-o", str(so),
                    str(tmp_path / "m.c"), "-lm"], check=True)
    import ctypes
    saved = oracle._lib
    oracle._lib = None
    try:
        real = oracle.lib()
        m = ctypes.CDLL(str(so))
        for fn in ("oracle_kv_write", "oracle_paged_decode", "oracle_paged_decode_partitioned",
                   "oracle_block_tokens"):
            getattr(m, fn).argtypes = getattr(real, fn).argtypes
            getattr(m, fn).restype = getattr(real, fn).restype
        oracle._lib = m
        failures = 0
        for pin in (lambda: test_oracle_matches_library_attention(128, 8, 2, [16, 15, 47, 64]),
                    test_len_one_returns_v_exactly, test_two_keys_logistic_weights):
            try:
                pin()
            except (AssertionError, ValueError):
                failures += 1
        assert failures >= 1, f"mutation '{name}' passed every pin"
    finally:
        oracle._lib = saved


def test_copy_on_write_beams_attend_to_their_own_tokens():
    """Beams forked mid-block (the parent's last block is partly filled) share
    the prefix blocks; each beam's next token triggers a private copy of the
    shared block.  Every beam must then attend to the shared prefix plus its
    own token only -- checked against torch fp64 attention on un-paged K/V."""
    d, hkv, hq = 64, 2, 4
    gen = wl.rng(31)
    prefix_k, prefix_v = rb((40, hkv, d), gen), rb((40, hkv, d), gen)
    nb = 32
    bm = BlockManager(nb, gen.permutation(nb))
    kc, vc = rb((nb, hkv, BT, d), gen), rb((nb, hkv, BT, d), gen)
    bm.add_seq(0, 0)
    slots = [bm.append_token(0) for _ in range(40)]
    kc, vc = oracle.kv_write(kc, vc, prefix_k, prefix_v, np.array(slots))
    for beam in (1, 2, 3):
        bm.fork(0, beam)
    beams = [0, 1, 2, 3]
    new_k, new_v = rb((4, hkv, d), gen), rb((4, hkv, d), gen)
    step_slots = np.array(bm.append_tokens(beams))
    src, dst = bm.take_copies()
    assert len(src) == 3 and len(set(dst.tolist())) == 3   # three beams copy, the last keeps it
    kc, vc = oracle.copy_blocks(kc, vc, src, dst)
    kc, vc = oracle.kv_write(kc, vc, new_k, new_v, step_slots)
    tables, lens = bm.export(beams, 3)
    q = rb((4, hq, d), gen)
    got = oracle.paged_decode(q, kc, vc, tables, lens, 0.125)
    ks = [np.concatenate([prefix_k, new_k[i:i + 1]]) for i in range(4)]
    vs = [np.concatenate([prefix_v, new_v[i:i + 1]]) for i in range(4)]
    np.testing.assert_allclose(got, sdpa_reference(q, ks, vs, 0.125), rtol=0, atol=1e-12)
    with pytest.raises(ValueError):
        oracle.copy_blocks(kc, vc, np.array([0]), np.array([nb]))


def test_swap_out_and_in_leaves_attention_unchanged():
    """Swap space: moving a sequence's blocks to host slots and back into
    other GPU blocks (with the freed blocks overwritten meanwhile) gives the
    same attention output, bit for bit."""
    w = wl.build("llama", 6, BlockManager, batch=5, len_lo=20, len_hi=90, head_dim=64,
                 poison=False, pool_factor=2.0)
    kc, vc = oracle.kv_write(w.k_cache, w.v_cache, w.k_new, w.v_new, w.slot_mapping)
    base = oracle.paged_decode(w.q, kc, vc, w.block_tables, w.lens, w.cfg["scale"])
    bm = w.alloc
    bm.set_host_pool(32)
    hk = np.zeros((32,) + kc.shape[1:], np.uint16)
    hv = np.zeros_like(hk)
    for s in (1, 3):
        bm.swap_out(s)
    g, h = bm.take_swaps(0)
    kc, vc, hk, hv = oracle.swap_blocks(kc, vc, hk, hv, g, h, 0)
    kc[g] = wl.BF16_NAN  # the freed blocks are reused meanwhile
    vc[g] = wl.BF16_NAN
    with pytest.raises(Exception):
        bm.append_token(1)  # a swapped-out sequence only comes back or is freed
    for s in (3, 1):
        bm.swap_in(s)
    g2, h2 = bm.take_swaps(1)
    assert sorted(h2.tolist()) == sorted(h.tolist())
    kc, vc, hk, hv = oracle.swap_blocks(kc, vc, hk, hv, g2, h2, 1)
    tables, lens = bm.export(list(range(5)), w.block_tables.shape[1])
    assert not np.array_equal(tables, w.block_tables)  # sequences 1 and 3 moved
    out = oracle.paged_decode(w.q, kc, vc, tables, lens, w.cfg["scale"])
    assert np.array_equal(out, base)


@pytest.mark.parametrize("hq,hkv,d,lens", [(4, 4, 64, [1, 37, 90]), (8, 2, 128, [20, 65])])
def test_prefill_matches_causal_library_attention(hq, hkv, d, lens):
    """Fresh prompts: the paged causal prefill equals torch's fp64 causal
    scaled_dot_product_attention on the un-paged K/V."""
    q, ks, vs = random_case(40 + d, lens, hq, hkv, d)
    gen = wl.rng(41)
    qrows = rb((sum(lens), hq, d), gen)
    kc, vc, tables, lens_ = page_sequences(ks, vs, 64, seed=42)
    qs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    got = oracle.paged_prefill(qrows, kc, vc, tables, lens_, qs, 0.125)
    for b, n in enumerate(lens):
        qt = torch.from_numpy(f32(qrows[qs[b]:qs[b + 1]])).permute(1, 0, 2)[None]   # [1, Hq, n, d]
        kt = torch.from_numpy(f32(ks[b])).permute(1, 0, 2)[None]
        vt = torch.from_numpy(f32(vs[b])).permute(1, 0, 2)[None]
        want = F.scaled_dot_product_attention(qt, kt, vt, is_causal=True, scale=0.125,
                                              enable_gqa=True)[0].permute(1, 0, 2).numpy()
        np.testing.assert_allclose(got[qs[b]:qs[b + 1]], want, rtol=0, atol=1e-12)


def test_prefill_after_cached_prefix_uses_an_offset_causal_mask():
    """A chunk of new tokens after cached ones: row i (position c + i) sees
    keys [0, c + i] -- torch attention with that explicit mask."""
    hq = hkv = 2
    d, ctx, new = 64, 75, 11
    q, ks, vs = random_case(43, [ctx], hq, hkv, d)
    qrows = rb((new, hq, d), wl.rng(44))
    kc, vc, tables, lens_ = page_sequences(ks, vs, 16, seed=45)
    got = oracle.paged_prefill(qrows, kc, vc, tables, lens_, np.array([0, new]), 0.3)
    pos = ctx - new + np.arange(new)
    mask = torch.from_numpy(np.arange(ctx)[None, :] <= pos[:, None])
    qt = torch.from_numpy(f32(qrows)).permute(1, 0, 2)[None]
    kt = torch.from_numpy(f32(ks[0])).permute(1, 0, 2)[None]
    vt = torch.from_numpy(f32(vs[0])).permute(1, 0, 2)[None]
    want = F.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=0.3)[0].permute(1, 0, 2)
    np.testing.assert_allclose(got, want.numpy(), rtol=0, atol=1e-12)
