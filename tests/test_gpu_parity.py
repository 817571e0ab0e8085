"""GPU parity: the CUDA write and decode kernels, called through the C ABI,
against the fp64 oracle on the same seeded inputs.

* write: the whole cache pool bit-exact against the oracle's write;
* decode: every output element within |err| <= 1e-2 + 1e-2 |ref|, for the
  single-pass and split-K variants, at sizes the oracle finishes in seconds
  (several blocks per partition, ragged tails) and at the full workload sizes
  (every sequence of every workload).
Free blocks, slots past each sequence's end and the new token's slot hold bf16
NaN before the write, so a stray read or a missed write shows up as NaN.
"""
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

SINGLE, SPLIT, CLUSTER = pkv.DECODE_SINGLE, pkv.DECODE_SPLIT, pkv.DECODE_CLUSTER


def test_tiny_end_to_end():
    w = build("tiny", 0)
    d = DeviceStep(w)
    d.write()
    kc, vc, ref = oracle_after_write(w)
    assert np.array_equal(host_bits(d.kc), kc) and np.array_equal(host_bits(d.vc), vc)
    for variant, part in ((SINGLE, 512), (SPLIT, 512), (SPLIT, 16), (SPLIT, 32), (CLUSTER, 512),
                          (CLUSTER, 16)):
        out = d.decode(variant, part)
        check_close(out, ref, f"tiny variant {variant} partition {part}")
    assert d.err_word() == 0


SMALL = [
    ("tiny", {}),
    ("llama", dict(batch=6, len_lo=1, len_hi=700)),
    ("qwen", dict(batch=5, len_lo=1, len_hi=1300)),
    ("prefix", dict(batch=4, prefix_len=512, suffix_lo=1, suffix_hi=90)),
    ("long", dict(batch=2, len_fixed=2600, num_blocks=400)),
    ("llama", dict(batch=5, head_dim=64, len_lo=1, len_hi=300)),
    ("qwen", dict(batch=4, head_dim=64, len_lo=1, len_hi=500)),
    ("qwen", dict(batch=3, num_heads=8, num_kv_heads=4, len_lo=1, len_hi=400)),   # group 2
    ("qwen", dict(batch=3, num_heads=32, num_kv_heads=4, len_lo=1, len_hi=400)),  # group 8
    ("qwen", dict(batch=3, num_heads=24, num_kv_heads=2, len_lo=1, len_hi=400)),  # group 12
    ("qwen", dict(batch=2, num_heads=16, num_kv_heads=1, len_lo=1, len_hi=300, head_dim=64)),
]


@pytest.mark.parametrize("name,kw", SMALL, ids=[f"{n}-{i}" for i, (n, _) in enumerate(SMALL)])
def test_parity_small(name, kw):
    w = build(name, 1, **kw)
    d = DeviceStep(w)
    d.write()
    kc, vc, ref = oracle_after_write(w)
    assert np.array_equal(host_bits(d.kc), kc), "write not bit-exact (K)"
    assert np.array_equal(host_bits(d.vc), vc), "write not bit-exact (V)"
    for variant, part in ((SINGLE, 512), (SPLIT, 512), (SPLIT, 64), (CLUSTER, 512), (CLUSTER, 64),
                          (pkv.DECODE_AUTO, 512)):
        check_close(d.decode(variant, part), ref, f"{name} {kw} variant {variant}/{part}")
    assert d.err_word() == 0


FULL = ["llama", "qwen", "prefix", "long"]


@pytest.mark.parametrize("name", FULL)
def test_parity_full_size(name):
    """Every output row of the full workload against the oracle (all host
    threads), in every variant, after a bit-exact write of the whole pool."""
    w = build(name, 0)
    d = DeviceStep(w)
    d.write()
    kc, vc, ref = oracle_after_write(w)
    assert np.array_equal(host_bits(d.kc), kc) and np.array_equal(host_bits(d.vc), vc)
    for variant in (pkv.DECODE_AUTO, SINGLE, SPLIT, CLUSTER):
        check_close(d.decode(variant, 512), ref, f"{name} full, variant {variant}")
    assert d.err_word() == 0


def test_len_one_is_v_exactly():
    w = build("qwen", 2, batch=4, len_lo=1, len_hi=1)
    d = DeviceStep(w)
    d.write()
    g = w.cfg["num_heads"] // w.cfg["num_kv_heads"]
    for variant in (SINGLE, SPLIT, CLUSTER):
        out = d.decode(variant, 512)
        assert np.array_equal(out, np.repeat(w.v_new, g, axis=1))
    w = build("llama", 2, batch=3, len_lo=1, len_hi=1)
    d = DeviceStep(w)
    d.write()
    assert np.array_equal(d.decode(SINGLE), w.v_new)
    assert np.array_equal(d.decode(CLUSTER, 16), w.v_new)


def test_block_relabelling_is_bit_exact_on_gpu():
    for name, kw in (("qwen", dict(batch=4, len_lo=20, len_hi=900)),
                     ("llama", dict(batch=4, len_lo=20, len_hi=900))):
        w = build(name, 3, **kw)
        d = DeviceStep(w)
        d.write()
        outs = {v: d.decode(v, 128) for v in (SINGLE, SPLIT, CLUSTER)}
        perm = wl.rng(4).permutation(w.num_blocks)
        t2, s2, kc2, vc2 = permute_pool(perm, w.block_tables, w.slot_mapping,
                                           host_bits(d.kc), host_bits(d.vc))
        d2 = DeviceStep(w)
        d2.kc.copy_(torch.from_numpy(kc2.view(np.int16)).view(torch.bfloat16))
        d2.vc.copy_(torch.from_numpy(vc2.view(np.int16)).view(torch.bfloat16))
        d2.tables = torch.from_numpy(t2).cuda()
        for v in (SINGLE, SPLIT, CLUSTER):
            assert np.array_equal(d2.decode(v, 128), outs[v])


def test_shared_prefix_matches_private_copy_on_gpu():
    w = build("prefix", 4, batch=6, prefix_len=320, suffix_lo=1, suffix_hi=60)
    d = DeviceStep(w)
    d.write()
    base = d.decode(SPLIT, 128)
    nb, npre = w.num_blocks, 20
    shared = w.block_tables[0, :npre]
    assert (w.block_tables[:, :npre] == shared).all()
    kc = host_bits(d.kc)
    vc = host_bits(d.vc)
    kc2 = np.concatenate([kc] + [kc[shared]] * 6)
    vc2 = np.concatenate([vc] + [vc[shared]] * 6)
    t2 = w.block_tables.copy()
    for b in range(6):
        t2[b, :npre] = nb + npre * b + np.arange(npre)
    d2 = DeviceStep(w)
    d2.kc = torch.from_numpy(kc2.view(np.int16)).view(torch.bfloat16).cuda()
    d2.vc = torch.from_numpy(vc2.view(np.int16)).view(torch.bfloat16).cuda()
    d2.tables = torch.from_numpy(t2).cuda()
    assert np.array_equal(d2.decode(SPLIT, 128), base)
    assert np.array_equal(d2.decode(CLUSTER, 64), d.decode(CLUSTER, 64))


CLUSTER_SHAPES = [
    # (workload, overrides, partition): parts per sequence = the longest table / partition, <= 8
    ("llama", dict(batch=200, len_lo=1, len_hi=40, head_dim=64), 16),      # 3 parts, many clusters
    ("long", dict(batch=1, len_fixed=32768), 512),                         # 8 parts of 256 blocks
    ("qwen", dict(batch=3, len_lo=1, len_hi=300), 16),                     # short rows: empty parts
    ("qwen", dict(batch=1, len_lo=1, len_hi=1), 16),                       # one block, one part
    ("qwen", dict(batch=40, len_lo=1, len_hi=300, num_heads=24, num_kv_heads=2), 64),  # 2 chunks
    ("qwen", dict(batch=7, len_lo=100, len_hi=900, head_dim=64, num_heads=16, num_kv_heads=2), 32),
]


AUTO_SPLIT_SHAPES = [
    # shapes where the automatic choice takes split-K (more units than one
    # wave holds in clusters of two, or cluster parts too long)
    ("llama", dict(batch=9, len_lo=1, len_hi=700)),                          # 288 units
    ("llama", dict(batch=8, len_lo=1, len_hi=2048, head_dim=64)),
    ("long", dict(batch=2, len_fixed=32768)),                                # 2 x 2048 blocks
    ("long", dict(batch=3, len_lo=1, len_hi=20000)),                         # ragged long rows
    ("qwen", dict(batch=60, len_lo=1, len_hi=4096)),                         # GQA, 240 units
    ("llama", dict(batch=12, len_lo=1, len_hi=1200)),
]


@pytest.mark.parametrize("name,kw", AUTO_SPLIT_SHAPES,
                         ids=[f"{n}-{i}" for i, (n, _) in enumerate(AUTO_SPLIT_SHAPES)])
def test_auto_split_shapes(name, kw):
    """Split-K through the automatic choice, against the oracle and bit for
    bit against the explicit split-K call with the partials' bytes only."""
    w = build(name, 5, **kw)
    c = w.cfg
    W = w.block_tables.shape[1]
    args = (c["batch"], c["num_heads"], c["num_kv_heads"], c["head_dim"], W)
    need = pkv.decode_workspace_bytes_for(pkv.DECODE_AUTO, *args, 512)
    assert pkv.decode_variant_for(*args, 512, need) == SPLIT
    split = pkv.decode_workspace_bytes(c["batch"], c["num_heads"], c["head_dim"], W, 512)
    assert need == max(split, (4 * c["batch"] + 255) // 256 * 256)
    d = DeviceStep(w)
    d.write()
    _, _, ref = oracle_after_write(w)
    auto = d.decode(pkv.DECODE_AUTO, 512)
    check_close(auto, ref, f"automatic split {name} {kw}")
    ws = torch.empty(split, dtype=torch.uint8, device="cuda")
    pkv.paged_attention_decode(d.out, d.q, d.kc, d.vc, d.tables, d.lens, c["scale"],
                               c["num_kv_heads"], variant=SPLIT, partition_tokens=512,
                               workspace=ws, err=d.err)
    assert np.array_equal(host_bits(d.out), auto)
    assert d.err_word() == 0


@pytest.mark.parametrize("name,kw,part", CLUSTER_SHAPES,
                         ids=[f"{n}-{i}" for i, (n, _, _) in enumerate(CLUSTER_SHAPES)])
def test_cluster_variant_shapes(name, kw, part):
    """The cluster variant where its parts are many, long, empty or single."""
    w = build(name, 11, **kw)
    d = DeviceStep(w)
    d.write()
    kc, vc, ref = oracle_after_write(w)
    out = d.decode(CLUSTER, part)
    check_close(out, ref, f"cluster {name} {kw} partition {part}")
    assert d.err_word() == 0


def test_longest_first_order_changes_nothing_but_scheduling():
    """The single-pass grid runs its units longest-first when the workspace can
    hold the order; the outputs are bit-identical to the unordered grid."""
    w = build("qwen", 15, batch=40, len_lo=1, len_hi=900)
    d = DeviceStep(w)
    d.write()
    ordered = d.decode(SINGLE)  # the binding supplies the workspace
    c = w.cfg
    rc = pkv.lib().pkv_paged_attention_decode_ex(
        d.out.data_ptr(), d.q.data_ptr(), d.kc.data_ptr(), d.vc.data_ptr(), d.tables.data_ptr(),
        d.tables.shape[1], d.lens.data_ptr(), c["batch"], c["num_heads"], c["num_kv_heads"],
        c["head_dim"], w.num_blocks, c["scale"], SINGLE, 512, None, 0, None,
        torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert rc == pkv.OK
    assert np.array_equal(host_bits(d.out), ordered)
