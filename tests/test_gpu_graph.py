"""The step's kernels captured in a CUDA graph and replayed (how serving
engines run decode): a replay gives bit-identical outputs to direct calls,
also after the inputs change in place between replays.  Covers the write +
decode step (every decode variant; the single pass launches its longest-first
order kernel and the split-K pass its merge as dependent launches), the
shared-prefix cascade and the tcgen05 prefill."""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import DeviceStep, build, check_close, dev_bf16, host_bits

pytestmark = pytest.mark.gpu
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from paged_kv_cache_459_b200 import pkv  # noqa: E402
import workloads as wl  # noqa: E402


def capture(step):
    """Warm the step up on a side stream, then capture it; returns the graph."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    return g


def same(a: torch.Tensor, b: torch.Tensor) -> bool:
    return torch.equal(a.view(torch.int16), b.view(torch.int16))


@pytest.mark.parametrize("variant", [pkv.DECODE_AUTO, pkv.DECODE_SINGLE, pkv.DECODE_SPLIT,
                                     pkv.DECODE_CLUSTER])
def test_decode_step_replays_from_a_graph(variant):
    w = build("qwen", 4, batch=12, len_lo=40, len_hi=1200)
    d = DeviceStep(w)
    c = w.cfg
    B, hq, hkv, dh = c["batch"], c["num_heads"], c["num_kv_heads"], c["head_dim"]
    W = w.block_tables.shape[1]
    ws = torch.empty(max(pkv.decode_workspace_bytes_for(variant, B, hq, hkv, dh, W, 512), 256),
                     dtype=torch.uint8, device="cuda")
    out_g = torch.zeros_like(d.q)

    def step(out):
        pkv.paged_kv_write(d.k_new, d.v_new, d.kc, d.vc, d.slots, err=d.err)
        pkv.paged_attention_decode(out, d.q, d.kc, d.vc, d.tables, d.lens, c["scale"], hkv,
                                   variant=variant, partition_tokens=512, workspace=ws, err=d.err)

    g = capture(lambda: step(out_g))
    out_g.zero_()
    g.replay()
    out_d = torch.empty_like(d.q)
    step(out_d)
    torch.cuda.synchronize()
    assert same(out_g, out_d)
    kc, vc = oracle.kv_write(w.k_cache, w.v_cache, w.k_new, w.v_new, w.slot_mapping)
    ref = oracle.paged_decode(w.q, kc, vc, w.block_tables, w.lens, c["scale"])
    check_close(host_bits(out_g), ref, f"graph replay, variant {variant}")
    # new queries written in place: the replay reads them
    q2 = wl.bf16_normal(w.q.shape, 77, 0)
    d.q.copy_(dev_bf16(q2))
    g.replay()
    step(out_d)
    torch.cuda.synchronize()
    assert same(out_g, out_d)
    ref2 = oracle.paged_decode(q2, kc, vc, w.block_tables, w.lens, c["scale"])
    check_close(host_bits(out_g), ref2, f"graph replay after new q, variant {variant}")
    assert d.err_word() == 0


@pytest.mark.parametrize("variant", [pkv.DECODE_SINGLE, pkv.DECODE_SPLIT])
def test_fused_step_replays_from_a_graph(variant):
    w = build("llama", 8, batch=10, len_lo=30, len_hi=900)
    d = DeviceStep(w)
    c = w.cfg
    B, hq, hkv, dh = c["batch"], c["num_heads"], c["num_kv_heads"], c["head_dim"]
    W = w.block_tables.shape[1]
    ws = torch.empty(max(pkv.decode_workspace_bytes_for(variant, B, hq, hkv, dh, W, 512), 256),
                     dtype=torch.uint8, device="cuda")
    out_g = torch.zeros_like(d.q)

    def step(out):
        pkv.paged_decode_step(out, d.q, d.k_new, d.v_new, d.kc, d.vc, d.tables, d.lens, c["scale"],
                              hkv, variant=variant, partition_tokens=512, workspace=ws, err=d.err)

    g = capture(lambda: step(out_g))
    out_g.zero_()
    g.replay()
    out_d = torch.empty_like(d.q)
    step(out_d)
    torch.cuda.synchronize()
    assert same(out_g, out_d)
    kc, vc = oracle.kv_write(w.k_cache, w.v_cache, w.k_new, w.v_new, w.slot_mapping)
    assert np.array_equal(host_bits(d.kc), kc) and np.array_equal(host_bits(d.vc), vc)
    ref = oracle.paged_decode(w.q, kc, vc, w.block_tables, w.lens, c["scale"])
    check_close(host_bits(out_g), ref, f"fused step graph replay, variant {variant}")
    assert d.err_word() == 0


def test_cascade_replays_from_a_graph():
    w = build("prefix", 5, batch=12, prefix_len=320, suffix_lo=1, suffix_hi=150, prefix_groups=2)
    d = DeviceStep(w)
    c = w.cfg
    B, hq, dh = c["batch"], c["num_heads"], c["head_dim"]
    W = w.block_tables.shape[1]
    pb_h, offs_h, mem_h = w.alloc.prefix_groups(list(range(B)))
    pb, offs, mem = (torch.from_numpy(np.ascontiguousarray(x, np.int32)).cuda() for x in (pb_h, offs_h, mem_h))
    bound = pkv.suffix_blocks_bound(w.lens, pb_h)
    ws = torch.empty(pkv.decode_prefix_workspace_bytes(B, hq, dh, W, 512), dtype=torch.uint8, device="cuda")
    out_g = torch.zeros_like(d.q)

    def step(out):
        pkv.paged_kv_write(d.k_new, d.v_new, d.kc, d.vc, d.slots, err=d.err)
        pkv.paged_attention_decode_prefix(out, d.q, d.kc, d.vc, d.tables, d.lens, c["scale"],
                                          c["num_kv_heads"], pb, offs, mem, max_suffix_blocks=bound,
                                          workspace=ws, err=d.err)

    g = capture(lambda: step(out_g))
    out_g.zero_()
    g.replay()
    out_d = torch.empty_like(d.q)
    step(out_d)
    torch.cuda.synchronize()
    assert same(out_g, out_d)
    kc, vc = oracle.kv_write(w.k_cache, w.v_cache, w.k_new, w.v_new, w.slot_mapping)
    ref = oracle.paged_decode(w.q, kc, vc, w.block_tables, w.lens, c["scale"])
    check_close(host_bits(out_g), ref, "cascade graph replay")
    assert d.err_word() == 0


def test_prefill_replays_from_a_graph():
    hq, hkv, dh, new = 16, 4, 128, [300, 77, 520]
    B = len(new)
    nb = sum(-(-n // 16) for n in new) + 8
    from oracle.alloc_model import BlockManager
    bm = BlockManager(nb, wl.rng(6).permutation(nb))
    for b in range(B):
        bm.add_seq(b, 0)
    slots = np.concatenate([bm.extend(b, new[b]) for b in range(B)])
    tables, lens = bm.export(list(range(B)), max(-(-n // 16) for n in new))
    kc = wl.bf16_normal((nb, hkv, 16, dh), 6, 0)
    vc = wl.bf16_normal((nb, hkv, 16, dh), 6, 1)
    T = sum(new)
    k_new, v_new = wl.bf16_normal((T, hkv, dh), 6, 2), wl.bf16_normal((T, hkv, dh), 6, 3)
    q = wl.bf16_normal((T, hq, dh), 6, 4)
    qs = np.concatenate([[0], np.cumsum(new)]).astype(np.int32)
    gk, gv, gq = dev_bf16(kc), dev_bf16(vc), dev_bf16(q)
    gkn, gvn = dev_bf16(k_new), dev_bf16(v_new)
    t_d, l_d, q_d = (torch.from_numpy(x).cuda() for x in (tables, lens, qs))
    s_d = torch.from_numpy(slots).cuda()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out_g = torch.zeros((T, hq, dh), dtype=torch.bfloat16, device="cuda")

    def step(out):
        pkv.paged_kv_write(gkn, gvn, gk, gv, s_d, err=err)
        pkv.paged_attention_prefill(out, gq, gk, gv, t_d, l_d, q_d, 1 / np.sqrt(dh), hkv, max(new), err=err)

    g = capture(lambda: step(out_g))
    out_g.zero_()
    g.replay()
    out_d = torch.empty_like(out_g)
    step(out_d)
    torch.cuda.synchronize()
    assert same(out_g, out_d)
    rk, rv = oracle.kv_write(kc, vc, k_new, v_new, slots)
    check_close(host_bits(out_g), oracle.paged_prefill(q, rk, rv, tables, lens, qs, 1 / np.sqrt(dh)),
                "prefill graph replay")
    assert int(err.item()) == 0
