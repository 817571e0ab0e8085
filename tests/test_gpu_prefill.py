"""GPU parity of the paged prefill path: the prompt's K/V written through the
allocator's slots (step 二 of the lifecycle: a new block as each one fills),
then causal attention of the prompt over the paged cache, against the fp64
oracle.  Covers fresh prompts, a chunk after cached tokens, grouped heads,
d = 64 and 128, NaN-poisoned free blocks and tail slots."""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import check_close, dev_bf16, host_bits
from oracle.alloc_model import BlockManager

pytestmark = pytest.mark.gpu
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from paged_kv_cache_459_b200 import pkv  # noqa: E402
import workloads as wl  # noqa: E402


def run_prefill(hq, hkv, d, cached, new, seed):
    """cached[b] tokens already in the cache, new[b] prompt tokens this call."""
    B = len(new)
    total = [c + n for c, n in zip(cached, new)]
    nb = sum(-(-t // 16) for t in total) + 8
    gen = wl.rng(seed)
    bm = BlockManager(nb, gen.permutation(nb))
    kc = wl.bf16_normal((nb, hkv, 16, d), seed, 0)
    vc = wl.bf16_normal((nb, hkv, 16, d), seed, 1)
    for b in range(B):
        bm.add_seq(b, cached[b])
    slots = np.concatenate([bm.extend(b, new[b]) for b in range(B)])
    tables, lens = bm.export(list(range(B)), max(-(-t // 16) for t in total))
    # poison: free blocks and slots past each sequence's end
    wl.poison_cache(kc, vc, np.array(bm.free_blocks()), tables, lens, np.array([], np.int64))
    T = sum(new)
    k_new, v_new = wl.bf16_normal((T, hkv, d), seed, 2), wl.bf16_normal((T, hkv, d), seed, 3)
    q = wl.bf16_normal((T, hq, d), seed, 4)
    qs = np.concatenate([[0], np.cumsum(new)]).astype(np.int32)
    scale = 1 / np.sqrt(d)
    rk, rv = oracle.kv_write(kc, vc, k_new, v_new, slots)
    ref = oracle.paged_prefill(q, rk, rv, tables, lens, qs, scale)

    gk, gv = dev_bf16(kc), dev_bf16(vc)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkv.paged_kv_write(dev_bf16(k_new), dev_bf16(v_new), gk, gv, torch.from_numpy(slots).cuda(), err=err)
    out = torch.empty((T, hq, d), dtype=torch.bfloat16, device="cuda")
    pkv.paged_attention_prefill(out, dev_bf16(q), gk, gv, torch.from_numpy(tables).cuda(),
                                torch.from_numpy(lens).cuda(), torch.from_numpy(qs).cuda(), scale, hkv,
                                max(new), err=err)
    torch.cuda.synchronize()
    assert np.array_equal(host_bits(gk), rk) and np.array_equal(host_bits(gv), rv)
    assert int(err.item()) == 0
    return host_bits(out), ref


@pytest.fixture
def prefill_impl():
    """The tcgen05/TMEM prefill kernel."""
    return "tcgen05"


@pytest.mark.parametrize("hq,hkv,d,cached,new", [
    (4, 4, 64, [0, 0, 0], [1, 37, 100]),
    (32, 32, 128, [0, 0], [300, 129]),
    (28, 4, 128, [0, 0, 0], [5, 64, 250]),
    (8, 2, 64, [200, 16, 0], [70, 1, 33]),       # chunks after cached tokens
    (16, 1, 128, [40], [90]),                      # one KV head, 16-query groups
    (8, 8, 128, [0, 1000], [700, 300]),            # several 64-key tiles, lazy rescaling
    (28, 4, 64, [0], [200]),                       # 1400 rows: several 128-row CTAs
])
def test_prefill_matches_oracle(hq, hkv, d, cached, new, prefill_impl):
    out, ref = run_prefill(hq, hkv, d, cached, new, seed=hq + d + len(new))
    check_close(out, ref, f"prefill {hq}/{hkv} d{d} cached {cached} new {new}")


def test_prefill_last_row_equals_decode(prefill_impl):
    """The prompt's last token attends exactly as a decode step at that length."""
    out, ref = run_prefill(8, 8, 128, [0], [77], seed=9)
    check_close(out[-1:], ref[-1:], "last row")


def test_prefill_many_items_ragged(prefill_impl):
    """More work items than SMs, with sequences whose last tile is partly or
    wholly empty and items past a short sequence's rows: each persistent CTA
    walks many items and all phases carry across them."""
    out, ref = run_prefill(32, 8, 128, [0, 500, 33, 0, 100, 0], [1500, 3, 700, 129, 1024, 257], seed=21)
    check_close(out, ref, "many items, ragged")


def test_prefill_full_size_sampled(prefill_impl):
    """The benchmark's size and launch (4 prompts x 2048 tokens, 32/32 heads,
    d 128), checked on a seeded sample of rows computed by the oracle one by one."""
    hq = hkv = 32
    d, B, n = 128, 4, 2048
    seed = 5
    nb = B * n // 16 + 8
    bm = BlockManager(nb, wl.rng(seed).permutation(nb))
    for b in range(B):
        bm.add_seq(b, 0)
    slots = np.concatenate([bm.extend(b, n) for b in range(B)])
    tables, lens = bm.export(list(range(B)), n // 16)
    kc = wl.bf16_normal((nb, hkv, 16, d), seed, 0)
    vc = wl.bf16_normal((nb, hkv, 16, d), seed, 1)
    T = B * n
    k_new, v_new = wl.bf16_normal((T, hkv, d), seed, 2), wl.bf16_normal((T, hkv, d), seed, 3)
    q = wl.bf16_normal((T, hq, d), seed, 4)
    qs = np.arange(0, T + 1, n, dtype=np.int32)
    scale = 1 / np.sqrt(d)
    gk, gv = dev_bf16(kc), dev_bf16(vc)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkv.paged_kv_write(dev_bf16(k_new), dev_bf16(v_new), gk, gv, torch.from_numpy(slots).cuda(), err=err)
    out = torch.empty((T, hq, d), dtype=torch.bfloat16, device="cuda")
    pkv.paged_attention_prefill(out, dev_bf16(q), gk, gv, torch.from_numpy(tables).cuda(),
                                torch.from_numpy(lens).cuda(), torch.from_numpy(qs).cuda(), scale, hkv,
                                n, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    rows = np.sort(wl.rng(seed + 1).choice(T, size=192, replace=False))
    rows = np.unique(np.concatenate([rows, [0, n - 1, n, T - 1]]))
    rk, rv = host_bits(gk), host_bits(gv)
    seq = rows // n
    ref = oracle.paged_decode(q[rows], rk, rv, tables[seq], (rows % n + 1).astype(np.int32), scale)
    check_close(host_bits(out)[rows], ref, "full-size sampled rows")


def test_prefill_many_items_d64(prefill_impl):
    """d = 64 with more work items than SMs (4-query groups, ragged prompts)."""
    out, ref = run_prefill(16, 4, 64, [0, 300, 0], [900, 17, 513], seed=31)
    check_close(out, ref, "many items, d 64")


def test_prefill_empty_prompts_in_batch(prefill_impl):
    """Sequences with no new tokens in the batch produce no rows and disturb
    nothing around them."""
    out, ref = run_prefill(8, 2, 128, [5, 0, 0, 20], [0, 37, 0, 130], seed=41)
    assert out.shape[0] == 167
    check_close(out, ref, "empty prompts in the batch")


def _prefill_case(hq, hkv, d, new, seed):
    B = len(new)
    nb = sum(-(-n // 16) for n in new) + 8
    bm = BlockManager(nb, wl.rng(seed).permutation(nb))
    for b in range(B):
        bm.add_seq(b, 0)
    slots = np.concatenate([bm.extend(b, new[b]) for b in range(B)])
    tables, lens = bm.export(list(range(B)), max(-(-n // 16) for n in new))
    kc = wl.bf16_normal((nb, hkv, 16, d), seed, 0)
    vc = wl.bf16_normal((nb, hkv, 16, d), seed, 1)
    T = sum(new)
    k_new, v_new = wl.bf16_normal((T, hkv, d), seed, 2), wl.bf16_normal((T, hkv, d), seed, 3)
    q = wl.bf16_normal((T, hq, d), seed, 4)
    qs = np.concatenate([[0], np.cumsum(new)]).astype(np.int32)
    rk, rv = oracle.kv_write(kc, vc, k_new, v_new, slots)
    return q, rk, rv, tables, lens, qs


def _run_gpu_prefill(q, rk, rv, tables, lens, qs, hkv, max_q):
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.zeros(q.shape, dtype=torch.bfloat16, device="cuda")
    pkv.paged_attention_prefill(out, dev_bf16(q), dev_bf16(rk), dev_bf16(rv), torch.from_numpy(tables).cuda(),
                                torch.from_numpy(lens).cuda(), torch.from_numpy(qs).cuda(),
                                1 / np.sqrt(q.shape[2]), hkv, max_q, err=err)
    torch.cuda.synchronize()
    return host_bits(out), int(err.item())


def test_prefill_inconsistent_length_is_flagged_and_skipped(prefill_impl):
    """A sequence whose context is shorter than its new tokens is skipped with
    the bad-length bit; the other sequences are unaffected."""
    new = [70, 90, 33]
    q, rk, rv, tables, lens, qs = _prefill_case(8, 8, 128, new, seed=51)
    ref = oracle.paged_prefill(q, rk, rv, tables, lens, qs, 1 / np.sqrt(128))
    bad = lens.copy()
    bad[1] = new[1] - 1
    out, err = _run_gpu_prefill(q, rk, rv, tables, bad, qs, 8, max(new))
    assert err & 4, err  # PKV_DEV_ERR_BAD_LEN
    keep = np.r_[qs[0]:qs[1], qs[2]:qs[3]]
    check_close(out[keep], ref[keep], "sequences next to a bad length")


def test_prefill_bad_table_entry_is_flagged(prefill_impl):
    """A table entry outside the pool is flagged (bad-block bit) and read as
    zeros; sequences that do not use it are unaffected."""
    new = [40, 100]
    q, rk, rv, tables, lens, qs = _prefill_case(8, 8, 64, new, seed=61)
    ref = oracle.paged_prefill(q, rk, rv, tables, lens, qs, 1 / np.sqrt(64))
    t = tables.copy()
    t[1, 2] = rk.shape[0] + 5
    out, err = _run_gpu_prefill(q, rk, rv, t, lens, qs, 8, max(new))
    assert err & 2, err  # PKV_DEV_ERR_BAD_BLOCK
    check_close(out[qs[0]:qs[1]], ref[qs[0]:qs[1]], "sequence next to a bad table entry")
