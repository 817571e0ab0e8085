"""GPU parity of the fused decode step (pkv_paged_decode_step): the new
token's K/V stored by the decode kernel itself, then attended.  Checked
against the oracle (cache bit-exact, output within tolerance) and against the
separate write + decode calls (bit-identical output), for every variant it
supports, ragged and full-size workloads, and its edge cases."""
import numpy as np
import pytest
import torch

from gpu_helpers import DeviceStep, build, check_close, host_bits, oracle_after_write

pytestmark = pytest.mark.gpu
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from paged_kv_cache_459_b200 import pkv  # noqa: E402
import workloads as wl  # noqa: E402

VARIANTS = [(pkv.DECODE_AUTO, 512), (pkv.DECODE_SINGLE, 512), (pkv.DECODE_SPLIT, 512),
            (pkv.DECODE_SPLIT, 64), (pkv.DECODE_CLUSTER, 512), (pkv.DECODE_CLUSTER, 32)]


def fused(d: DeviceStep, variant, part, kc=None, vc=None, tables=None, lens=None):
    kc = d.kc if kc is None else kc
    vc = d.vc if vc is None else vc
    pkv.paged_decode_step(d.out, d.q, d.k_new, d.v_new, kc, vc,
                          d.tables if tables is None else tables, d.lens if lens is None else lens,
                          d.w.cfg["scale"], d.w.cfg["num_kv_heads"], variant=variant,
                          partition_tokens=part, err=d.err)
    torch.cuda.synchronize()
    return host_bits(d.out)


CASES = [
    ("tiny", {}),
    ("llama", dict(batch=6, len_lo=1, len_hi=700)),
    ("qwen", dict(batch=5, len_lo=1, len_hi=1300)),
    ("long", dict(batch=2, len_fixed=2600, num_blocks=400)),
    ("qwen", dict(batch=4, head_dim=64, len_lo=1, len_hi=500)),
    ("qwen", dict(batch=3, num_heads=24, num_kv_heads=2, len_lo=1, len_hi=400)),  # 2 head chunks
]


@pytest.mark.parametrize("name,kw", CASES, ids=[f"{n}-{i}" for i, (n, _) in enumerate(CASES)])
def test_fused_step_matches_oracle_and_separate_calls(name, kw):
    w = build(name, 21, **kw)
    kc, vc, ref = oracle_after_write(w)
    for variant, part in VARIANTS:
        d = DeviceStep(w)   # fresh pre-write caches (NaN in the new tokens' slots)
        out = fused(d, variant, part)
        assert np.array_equal(host_bits(d.kc), kc), f"{name} {variant}: K cache"
        assert np.array_equal(host_bits(d.vc), vc), f"{name} {variant}: V cache"
        check_close(out, ref, f"{name} {kw} fused, variant {variant}/{part}")
        e = DeviceStep(w)
        e.write()
        assert np.array_equal(e.decode(variant, part), out), f"{name} {variant}: fused != separate"
        assert d.err_word() == 0


@pytest.mark.parametrize("name", ["llama", "qwen", "long"])
def test_fused_step_full_size(name):
    """The benchmark's step at full size: the whole pool bit-exact, every
    output row against the oracle, and the same bits as write + decode."""
    w = build(name, 0)
    d = DeviceStep(w)
    out = fused(d, pkv.DECODE_AUTO, 512)
    kc, vc, ref = oracle_after_write(w)
    assert np.array_equal(host_bits(d.kc), kc) and np.array_equal(host_bits(d.vc), vc)
    e = DeviceStep(w)
    e.write()
    assert np.array_equal(e.decode(pkv.DECODE_AUTO, 512), out)
    check_close(out, ref, f"{name} fused full size")
    assert d.err_word() == 0


def test_fused_step_zero_length_writes_nothing():
    w = build("llama", 22, batch=4, len_lo=30, len_hi=200)
    d = DeviceStep(w)
    lens = d.lens.clone()
    lens[2] = 0
    before_k, before_v = host_bits(d.kc), host_bits(d.vc)
    out = fused(d, pkv.DECODE_SINGLE, 512, lens=lens)
    slot = int(w.slot_mapping[2])
    blk, off = slot // 16, slot % 16
    assert np.array_equal(host_bits(d.kc)[blk, :, off], before_k[blk, :, off])
    assert np.array_equal(host_bits(d.vc)[blk, :, off], before_v[blk, :, off])
    assert (wl.bf16_to_f32(out[2]) == 0).all()


def test_fused_step_bad_last_block_is_flagged():
    w = build("llama", 23, batch=3, len_lo=40, len_hi=300)
    d = DeviceStep(w)
    t = d.tables.clone()
    last = (int(w.lens[1]) - 1) // 16
    t[1, last] = w.num_blocks + 3
    fused(d, pkv.DECODE_SINGLE, 512, tables=t)
    assert d.err_word() & 2  # PKV_DEV_ERR_BAD_BLOCK


def test_fused_step_refuses_an_unknown_variant():
    w = build("tiny", 24)
    d = DeviceStep(w)
    with pytest.raises(pkv.PkvError) as ex:
        fused(d, 3, 512)
    assert ex.value.code == pkv.ERR_INVALID_ARG


def test_prepared_step_matches_the_plain_call():
    """pkv.prepare_decode_step checks its tensors once; each call then runs the
    same library call on the same buffers: identical output and caches, and a
    change of the buffers' contents between calls is seen by the next call."""
    w = build("qwen", 25, batch=6, len_lo=1, len_hi=700)
    kc, vc, ref = oracle_after_write(w)
    d, e = DeviceStep(w), DeviceStep(w)
    out = fused(d, pkv.DECODE_AUTO, 512)
    step = pkv.prepare_decode_step(e.out, e.q, e.k_new, e.v_new, e.kc, e.vc, e.tables, e.lens,
                                   w.cfg["scale"], w.cfg["num_kv_heads"], err=e.err)
    step()
    torch.cuda.synchronize()
    assert np.array_equal(host_bits(e.out), out)
    assert np.array_equal(host_bits(e.kc), kc) and np.array_equal(host_bits(e.vc), vc)
    e.q.copy_(torch.flip(e.q, dims=[0]))  # new queries in the same buffer
    step()
    torch.cuda.synchronize()
    d.q.copy_(torch.flip(d.q, dims=[0]))
    assert np.array_equal(host_bits(e.out), fused(d, pkv.DECODE_AUTO, 512))
    assert e.err_word() == 0
