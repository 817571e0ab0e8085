"""The C++ block allocator against the reference model (oracle/alloc_model.py):
the pages' worked examples, random operation sequences compared step by step,
all-or-nothing failures, and the tables of every decode workload."""
import json
import os

import numpy as np
import pytest

from oracle.alloc_model import AllocError as ModelError, BlockManager
from paged_kv_cache_459_b200 import build as pkv_build
import workloads as wl

pkv_build.build()
from paged_kv_cache_459_b200.pkv import AllocError, BlockAllocator  # noqa: E402

BT = 16


def same_state(a: BlockAllocator, m: BlockManager, seq_ids):
    assert a.free_blocks() == m.free_blocks()
    assert [a.refcount(b) for b in range(m.num_blocks)] == m.ref
    ids = sorted(s for s in seq_ids if s not in m.swapped)
    if ids:
        w = max(1, max(len(m.tables[s]) for s in ids))
        ta, la = a.export(ids, w)
        tm, lm = m.export(ids, w)
        assert np.array_equal(ta, tm) and np.array_equal(la, lm)
    fa, ua, sa, xa = a.stats()
    fm, um, sm, xm = m.stats()
    assert (fa, ua, sa) == (fm, um, sm) and xa == pytest.approx(xm, abs=1e-12)


def test_sharing_example(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "sharing_example.json")))
    a = BlockAllocator(16, list(range(1, 16)) + [0])
    a.add_seq(0, 64)
    a.fork(0, 1, 48)
    for _ in range(16):
        a.append_token(1)
    a.fork(0, 2, 32)
    for _ in range(32):
        a.append_token(2)
    tables, _ = a.export([0, 1, 2], 4)
    assert tables.tolist() == [g["printed"]["tables"][k] for k in "ABC"]
    for blk, rc in g["expected_refcounts"].items():
        assert a.refcount(int(blk)) == rc
    a.free_seq(0)
    for blk, rc in g["expected_after_freeing_A"]["refcounts"].items():
        assert a.refcount(int(blk)) == rc
    assert a.free_blocks()[-1] == 4


def test_block_table_example(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "block_table_example.json")))
    t = g["printed"]["request_A_block_table"]
    order = [t["0"], t["1"], t["2"]] + [b for b in range(64) if b not in (t["0"], t["1"], t["2"])]
    a = BlockAllocator(64, order)
    a.add_seq(7, 0)
    slots = [a.append_token(7) for _ in range(48)]
    for tok, slot in g["expected_slot_by_token"].items():
        assert slots[int(tok) - 1] == slot == a.slot_of(7, int(tok) - 1)


@pytest.mark.parametrize("seed", range(6))
def test_random_operations_match_model(seed):
    gen = np.random.default_rng(seed)
    nb = int(gen.integers(8, 64))
    order = gen.permutation(nb)
    a, m = BlockAllocator(nb, order), BlockManager(nb, order)
    a.set_host_pool(24)
    m.set_host_pool(24)
    live, next_id = [], 0
    for step in range(400):
        op = gen.choice(["add", "append", "appends", "fork", "free", "out", "in"],
                        p=[.18, .3, .14, .14, .12, .06, .06])
        args = ()
        if op == "add":
            args = (next_id, int(gen.integers(0, 70)))
            next_id += 1
        elif op in ("append", "free", "out", "in") and live:
            args = (int(gen.choice(live)),)
        elif op == "appends" and live:
            k = int(gen.integers(1, len(live) + 1))
            args = (list(gen.choice(live, size=k, replace=False)),)
        elif op == "fork" and live:
            p = int(gen.choice(live))
            args = (p, next_id, int(gen.integers(-1, m.lens[p] + 2)))
            next_id += 1
        else:
            continue
        ra = rm = None
        ea = em = None
        try:
            ra = {"add": a.add_seq, "append": a.append_token, "appends": a.append_tokens,
                  "fork": a.fork, "free": a.free_seq, "out": a.swap_out, "in": a.swap_in}[op](*args)
        except AllocError as e:
            ea = e.kind
        try:
            rm = {"add": m.add_seq, "append": m.append_token, "appends": m.append_tokens,
                  "fork": m.fork, "free": m.free_seq, "out": m.swap_out, "in": m.swap_in}[op](*args)
            if op in ("append", "appends"):
                ca, cm = a.take_copies(), m.take_copies()
                assert all(np.array_equal(x, y) for x, y in zip(ca, cm)), (step, op)
            if op in ("out", "in"):
                d = 0 if op == "out" else 1
                sa, sm = a.take_swaps(d), m.take_swaps(d)
                assert all(np.array_equal(x, y) for x, y in zip(sa, sm)), (step, op)
        except ModelError as e:
            em = e.kind
        assert ea == em, (step, op, args, ea, em)
        if ea is None:
            if op in ("append", "appends"):
                assert list(np.atleast_1d(ra)) == list(np.atleast_1d(rm))
            if op in ("add", "fork"):
                live.append(args[1] if op == "fork" else args[0])
            if op == "free":
                live.remove(args[0])
        same_state(a, m, live)


def test_failures_change_nothing():
    a = BlockAllocator(4)
    a.add_seq(0, 40)
    before = (a.free_blocks(), [a.refcount(b) for b in range(4)], a.export([0], 3))
    for call in (lambda: a.add_seq(1, 33), lambda: a.add_seq(0, 1), lambda: a.fork(0, 0),
                 lambda: a.fork(5, 1), lambda: a.free_seq(9), lambda: a.fork(0, 1, 41),
                 lambda: a.append_tokens([0, 0]), lambda: a.append_tokens([0, 3])):
        with pytest.raises(AllocError):
            call()
        after = (a.free_blocks(), [a.refcount(b) for b in range(4)], a.export([0], 3))
        assert after[0] == before[0] and after[1] == before[1]
        assert np.array_equal(after[2][0], before[2][0])
    a.fork(0, 1)  # shares the partly filled third block
    a.add_seq(2, 16)  # takes the last free block
    before = (a.free_blocks(), [a.refcount(b) for b in range(4)])
    for call in (lambda: a.append_token(1), lambda: a.append_tokens([2]),
                 lambda: a.append_tokens([0, 1])):  # copy-on-write / new block: pool empty
        with pytest.raises(AllocError) as e:
            call()
        assert e.value.kind == "oom"
        assert (a.free_blocks(), [a.refcount(b) for b in range(4)]) == before
    a.free_seq(2)
    # sequence 0 comes first: it takes the copy; sequence 1 then holds the old block alone
    assert a.append_tokens([0, 1]).tolist()[0] == a.slot_of(0, 40)
    src, dst = a.take_copies()
    assert src.tolist() == [a.export([1], 3)[0][0, 2]] and dst.tolist() == [a.export([0], 3)[0][0, 2]]
    with pytest.raises(AllocError):
        BlockAllocator(3, [0, 1, 1])


@pytest.mark.parametrize("seed", range(4))
def test_append_into_keeps_the_host_tables_equal_to_export(seed):
    """The in-place batch append against a twin allocator driven by the plain
    batch append: the same slots and copy-on-write pairs, and the caller's
    tables and lengths equal to a fresh export after every step."""
    gen = np.random.default_rng(100 + seed)
    nb, width = 800, 40
    order = gen.permutation(nb)
    a, b = BlockAllocator(nb, order), BlockAllocator(nb, order)
    ids = list(range(6))
    for s in ids:
        n = int(gen.integers(0, 60))
        a.add_seq(s, n)
        b.add_seq(s, n)
    tables, lens = a.export(ids, width)
    next_id, cows = len(ids), 0
    for step in range(200):
        if gen.random() < 0.06:  # a fork, often mid-block: the child's next append copies
            p = int(gen.choice(ids))
            n = int(gen.integers(0, a.seq_len(p) + 1))
            a.fork(p, next_id, n)
            b.fork(p, next_id, n)
            ids.append(next_id)
            next_id += 1
            tables, lens = a.export(ids, width)  # a new set of sequences: export again
        sa = a.append_tokens_into(ids, tables, lens)
        sb = b.append_tokens(ids)
        assert sa.tolist() == sb.tolist(), step
        ca, cb = a.take_copies(), b.take_copies()
        assert all(np.array_equal(x, y) for x, y in zip(ca, cb)), step
        cows += len(ca[0])
        t2, l2 = a.export(ids, width)
        assert np.array_equal(tables, t2) and np.array_equal(lens, l2), step
    assert cows > 0 and len(ids) > 6


def test_append_into_errors_change_nothing():
    a = BlockAllocator(8)
    a.add_seq(0, 32)  # two full blocks: its next token needs a third
    a.add_seq(1, 5)
    tables, lens = a.export([0, 1], 2)
    keep = (tables.copy(), lens.copy(), a.free_blocks())
    for call in (lambda: a.append_tokens_into([0, 1], tables, lens),   # 0 would pass width 2
                 lambda: a.append_tokens_into([1, 1], tables, lens),   # named twice
                 lambda: a.append_tokens_into([1, 7], tables, lens),   # unknown sequence
                 lambda: a.append_tokens_into([0], tables, lens),      # rows != sequences
                 lambda: a.append_tokens_into([0, 1], tables.astype(np.int64), lens),
                 lambda: a.append_tokens_into([0, 1], tables[:, :1], lens)):  # not contiguous
        with pytest.raises(AllocError):
            call()
        assert np.array_equal(tables, keep[0]) and np.array_equal(lens, keep[1])
        assert a.free_blocks() == keep[2]
    b = BlockAllocator(2)
    b.add_seq(0, 16)
    b.add_seq(1, 16)  # both blocks full, the pool empty
    t, ln = b.export([0, 1], 4)
    k = (t.copy(), ln.copy())
    with pytest.raises(AllocError) as e:
        b.append_tokens_into([0, 1], t, ln)
    assert e.value.kind == "oom" and np.array_equal(t, k[0]) and np.array_equal(ln, k[1])


@pytest.mark.parametrize("name,kw", [("tiny", {}), ("llama", {}), ("qwen", {}), ("prefix", {}),
                                     ("long", {})])
def test_workload_tables_match_model(name, kw):
    w1 = wl.build(name, 0, BlockAllocator, with_cache=False, **kw)
    w2 = wl.build(name, 0, BlockManager, with_cache=False, **kw)
    assert np.array_equal(w1.block_tables, w2.block_tables)
    assert np.array_equal(w1.slot_mapping, w2.slot_mapping)
    assert np.array_equal(w1.lens, w2.lens)
    assert w1.free_blocks.tolist() == w2.free_blocks.tolist()
    if name == "prefix":
        assert all(w1.alloc.refcount(int(b)) == w1.cfg["batch"] for b in w1.block_tables[0, :125])
        assert w1.alloc.stats()[2] == 125


def test_prefix_groups_sharing_example(golden_dir):
    """The pages' example: blocks 1 and 2 are shared by all three tables."""
    g = json.load(open(os.path.join(golden_dir, "sharing_example.json")))
    for alloc_cls in (BlockAllocator, BlockManager):
        a = alloc_cls(16, list(range(1, 16)) + [0])
        a.add_seq(0, 64)
        a.fork(0, 1, 48)
        for _ in range(16):
            a.append_token(1)
        a.fork(0, 2, 32)
        for _ in range(32):
            a.append_token(2)
        pb, offs, members = a.prefix_groups([0, 1, 2])
        assert pb.tolist() == [len(g["printed"]["shared_by_three"])] * 3
        assert offs.tolist() == [0, 3] and members.tolist() == [0, 1, 2]


@pytest.mark.parametrize("kw", [dict(batch=12), dict(batch=20, prefix_groups=3, unshared_every=4),
                                dict(batch=9, prefix_len=48, suffix_lo=1, suffix_hi=30)])
def test_prefix_groups_match_model(kw):
    w1 = wl.build("prefix", 3, BlockAllocator, with_cache=False, **kw)
    w2 = wl.build("prefix", 3, BlockManager, with_cache=False, **kw)
    ids = list(range(w1.cfg["batch"]))
    r1, r2 = w1.alloc.prefix_groups(ids), w2.alloc.prefix_groups(ids)
    for x, y in zip(r1, r2):
        assert np.array_equal(x, y)
    pb, offs, members = r1
    groups = kw.get("prefix_groups", 1)
    assert len(offs) - 1 == groups
    # a member's prefix is the shared full blocks; 2000 tokens = 125 blocks
    for gi in range(groups):
        mem = members[offs[gi]:offs[gi + 1]]
        assert (pb[mem] == min(w1.cfg["prefix_len"], int(w1.lens[mem].min())) // 16).all()
        rows = w1.block_tables[mem, :pb[mem[0]]]
        assert (rows == rows[0]).all()


def test_prefix_groups_random_forks_match_model():
    gen = np.random.default_rng(5)
    for trial in range(20):
        nb = 200
        order = gen.permutation(nb)
        a, m = BlockAllocator(nb, order), BlockManager(nb, order)
        n0 = int(gen.integers(0, 90)) if trial % 2 else 64
        for x in (a, m):
            x.add_seq(0, n0)
        live = [0]
        r = np.random.default_rng(trial)
        for s in range(1, 12):
            parent = int(r.choice(live))
            n = int(r.integers(0, m.lens[parent] + 1))
            ext = int(r.integers(0, 40))
            for x in (a, m):
                x.fork(parent, s, n)
            try:
                for _ in range(ext):
                    for x in (a, m):
                        x.append_token(s)
            except Exception:
                pass
            live.append(s)
        ids = list(range(12))
        for x, y in zip(a.prefix_groups(ids), m.prefix_groups(ids)):
            assert np.array_equal(x, y)


def test_extend_matches_model_and_takes_blocks_as_they_fill():
    for alloc_cls in (BlockAllocator, BlockManager):
        a = alloc_cls(16, list(range(16)))
        a.add_seq(0, 0)
        slots = a.extend(0, 40)  # a 40-token prompt: blocks 0, 1, 2
        assert slots.tolist() == list(range(40))
        a.fork(0, 1)  # shares the partly filled third block
        s2 = a.extend(1, 30)  # copy-on-write first, then blocks as they fill
        assert s2[0] == 3 * 16 + 8 and a.take_copies()[0].tolist() == [2]
        with pytest.raises(Exception):
            a.extend(1, 16 * 20)  # not enough blocks: nothing changes
        n = a.seq_len(1) if hasattr(a, "seq_len") else a.lens[1]
        assert n == 70
