"""GPU parity of the shared-prefix (cascade) decode: the prefix blocks that a
group of block tables share are read once per (group, KV head); the result
must match the fp64 oracle, which reads every sequence's blocks on its own."""
import numpy as np
import pytest
import torch

from gpu_helpers import DeviceStep, build, check_close, host_bits, oracle_after_write

pytestmark = pytest.mark.gpu
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from paged_kv_cache_459_b200 import pkv  # noqa: E402
import workloads as wl  # noqa: E402
from relabel import permute_pool  # noqa: E402


def cascade(d: DeviceStep, part=512, tables=None, bound=0):
    """bound: max_suffix_blocks (0: unknown, "exact": from the host lengths)."""
    w = d.w
    pb, offs, members = w.alloc.prefix_groups(list(range(w.cfg["batch"])))
    if bound == "exact":
        bound = pkv.suffix_blocks_bound(w.lens, pb)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.int32)).cuda()  # noqa: E731
    pkv.paged_attention_decode_prefix(d.out, d.q, d.kc, d.vc, d.tables if tables is None else tables,
                                      d.lens, w.cfg["scale"], w.cfg["num_kv_heads"], dev(pb),
                                      dev(offs), dev(members), max_suffix_blocks=bound,
                                      partition_tokens=part, err=d.err)
    torch.cuda.synchronize()
    return host_bits(d.out), pb, offs


CASES = [
    ("prefix", dict(batch=6, prefix_len=320, suffix_lo=1, suffix_hi=60)),
    ("prefix", dict(batch=20, prefix_len=160, suffix_lo=1, suffix_hi=200, prefix_groups=3,
                    unshared_every=4)),
    ("prefix", dict(batch=9, prefix_len=208, suffix_lo=1, suffix_hi=100, num_heads=28,
                    num_kv_heads=4)),
    ("prefix", dict(batch=7, prefix_len=144, suffix_lo=1, suffix_hi=90, head_dim=64,
                    num_heads=16, num_kv_heads=2)),
    ("prefix", dict(batch=40, prefix_len=16, suffix_lo=1, suffix_hi=20)),   # one shared block
    ("prefix", dict(batch=5, prefix_len=1008, suffix_lo=1, suffix_hi=60)),  # two spans, 32 + 31 blocks
    # 280 rows (three row tiles) over two spans, grouped heads
    ("prefix", dict(batch=40, prefix_len=704, suffix_lo=1, suffix_hi=30, num_heads=28,
                    num_kv_heads=4)),
    ("prefix", dict(batch=5, prefix_len=48, suffix_lo=1, suffix_hi=1)),     # suffix = new token
    # more than 128 rows per (group, KV head): several row tiles, the last one ragged
    ("prefix", dict(batch=40, prefix_len=272, suffix_lo=1, suffix_hi=40, num_heads=28,
                    num_kv_heads=4)),                                        # 280 rows, chunks 8+8+1
    ("prefix", dict(batch=33, prefix_len=144, suffix_lo=1, suffix_hi=30, head_dim=64,
                    num_heads=8, num_kv_heads=2)),                           # 132 rows, d 64
]


@pytest.mark.parametrize("name,kw", CASES, ids=[str(i) for i in range(len(CASES))])
def test_cascade_matches_oracle(name, kw):
    w = build(name, 13, **kw)
    d = DeviceStep(w)
    d.write()
    kc, vc, ref = oracle_after_write(w)
    for part in (512, 64):
        for bound in (0, "exact"):
            out, pb, offs = cascade(d, part, bound=bound)
            assert len(offs) - 1 == kw.get("prefix_groups", 1) and pb.max() > 0
            check_close(out, ref, f"cascade {kw} partition {part} suffix bound {bound}")
    assert d.err_word() == 0


def test_cascade_suffix_bound_too_small_is_flagged():
    """A max_suffix_blocks below a real suffix leaves it incomplete and sets the
    bad-length bit (no out-of-range workspace use)."""
    w = build("prefix", 13, **CASES[1][1])
    d = DeviceStep(w)
    d.write()
    cascade(d, 64, bound=1)   # 4-block partitions: one covers 4 of up to 13 suffix blocks
    assert d.err_word() & 4


def test_cascade_full_size():
    """The prefix workload at full size (128 sequences sharing a 2000-token
    prefix): every output row against the oracle."""
    w = build("prefix", 0)
    d = DeviceStep(w)
    d.write()
    kc, vc, ref = oracle_after_write(w)
    assert np.array_equal(host_bits(d.kc), kc) and np.array_equal(host_bits(d.vc), vc)
    out, pb, offs = cascade(d, bound="exact")
    assert (pb == 125).all() and len(offs) == 2
    check_close(out, ref, "cascade full size")
    assert d.err_word() == 0


def test_cascade_block_relabelling_is_bit_exact():
    w = build("prefix", 14, batch=10, prefix_len=256, suffix_lo=1, suffix_hi=80, prefix_groups=2)
    d = DeviceStep(w)
    d.write()
    base, _, _ = cascade(d)
    perm = wl.rng(3).permutation(w.num_blocks)
    t2, _, kc2, vc2 = permute_pool(perm, w.block_tables, w.slot_mapping, host_bits(d.kc),
                                      host_bits(d.vc))
    d.kc.copy_(torch.from_numpy(kc2.view(np.int16)).view(torch.bfloat16))
    d.vc.copy_(torch.from_numpy(vc2.view(np.int16)).view(torch.bfloat16))
    out, _, _ = cascade(d, tables=torch.from_numpy(t2).cuda())
    assert np.array_equal(out, base)


@pytest.mark.parametrize("idx", [0, 1, 2, 3])
def test_cascade_fused_step(idx):
    """pkv_paged_decode_prefix_step: the step's write fused into the cascade --
    caches bit-exact with the oracle's write, output within tolerance, and
    bit-identical to the separate write + cascade."""
    name, kw = CASES[idx]
    w = build(name, 31, **kw)
    kc, vc, ref = oracle_after_write(w)
    pb, offs, members = w.alloc.prefix_groups(list(range(w.cfg["batch"])))
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.int32)).cuda()  # noqa: E731
    bound = pkv.suffix_blocks_bound(w.lens, pb)
    d = DeviceStep(w)
    pkv.paged_decode_prefix_step(d.out, d.q, d.k_new, d.v_new, d.kc, d.vc, d.tables, d.lens,
                                 w.cfg["scale"], w.cfg["num_kv_heads"], dev(pb), dev(offs),
                                 dev(members), max_suffix_blocks=bound, err=d.err)
    torch.cuda.synchronize()
    assert np.array_equal(host_bits(d.kc), kc) and np.array_equal(host_bits(d.vc), vc)
    out = host_bits(d.out)
    check_close(out, ref, f"fused cascade step {kw}")
    e = DeviceStep(w)
    e.write()
    sep, _, _ = cascade(e, bound="exact")
    assert np.array_equal(out, sep)
    assert d.err_word() == 0


def test_cascade_fused_step_token_inside_prefix_is_flagged():
    """A prefix_blocks entry that covers a sequence's last block (not what the
    allocator's grouping produces) leaves the fused write undone, flagged."""
    w = build("prefix", 32, batch=4, prefix_len=64, suffix_lo=16, suffix_hi=16)  # len 80: 5 full blocks
    pb, offs, members = w.alloc.prefix_groups(list(range(w.cfg["batch"])))
    pb = pb.copy()
    pb[1] = int(w.lens[1]) // 16      # claims the whole sequence, its new token included
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.int32)).cuda()  # noqa: E731
    d = DeviceStep(w)
    pkv.paged_decode_prefix_step(d.out, d.q, d.k_new, d.v_new, d.kc, d.vc, d.tables, d.lens,
                                 w.cfg["scale"], w.cfg["num_kv_heads"], dev(pb), dev(offs),
                                 dev(members), err=d.err)
    assert d.err_word() & 4
