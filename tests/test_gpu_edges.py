"""GPU edge cases: empty sequences, bad data caught on the device (flagged in
the error word, skipped, never trapping), skipped and out-of-range slots."""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import DeviceStep, bits_to_f64, build, check_close, host_bits

pytestmark = pytest.mark.gpu
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from paged_kv_cache_459_b200 import pkv  # noqa: E402

VARIANTS = [(pkv.DECODE_SINGLE, 512), (pkv.DECODE_SPLIT, 32), (pkv.DECODE_CLUSTER, 32)]


@pytest.mark.parametrize("name", ["llama", "qwen"])
def test_zero_length_sequence_gives_zero_row(name):
    w = build(name, 5, batch=4, len_lo=1, len_hi=120, head_dim=64)
    d = DeviceStep(w)
    d.write()
    kc, vc = oracle.kv_write(w.k_cache, w.v_cache, w.k_new, w.v_new, w.slot_mapping)
    lens = w.lens.copy()
    lens[2] = 0
    ref = oracle.paged_decode(w.q, kc, vc, w.block_tables, lens, w.cfg["scale"])
    for v, part in VARIANTS:
        out = d.decode(v, part, lens=torch.from_numpy(lens).cuda())
        assert (out[2] == 0).all()
        check_close(out, ref, f"zero-length, variant {v}")
    assert d.err_word() == 0


@pytest.mark.parametrize("name", ["llama", "qwen"])
def test_bad_table_entry_is_flagged_and_skipped(name):
    w = build(name, 6, batch=4, len_lo=40, len_hi=200)
    d = DeviceStep(w)
    d.write()
    kc, vc = oracle.kv_write(w.k_cache, w.v_cache, w.k_new, w.v_new, w.slot_mapping)
    ref = oracle.paged_decode(w.q, kc, vc, w.block_tables, w.lens, w.cfg["scale"])
    for bad in (w.num_blocks, w.num_blocks + 1000, -5, 2**31 - 1):
        t = w.block_tables.copy()
        t[1, 1] = bad
        d.err.zero_()
        for v, part in VARIANTS:
            out = d.decode(v, part, tables=torch.from_numpy(t).cuda())
            assert np.isfinite(bits_to_f64(out)).all()
            keep = [0, 2, 3]
            check_close(out[keep], ref[keep], f"rows beside a bad table entry, variant {v}")
        assert d.err_word() & pkv.DEV_ERR_BAD_BLOCK


def test_length_past_the_table_is_clamped_and_flagged():
    w = build("llama", 7, batch=3, len_lo=20, len_hi=60, head_dim=64)
    d = DeviceStep(w)
    d.write()
    lens = w.lens.copy()
    lens[0] = w.block_tables.shape[1] * 16 + 5
    lens[1] = -3
    for v, part in VARIANTS:
        d.err.zero_()
        out = d.decode(v, part, lens=torch.from_numpy(lens).cuda())
        assert d.err_word() & pkv.DEV_ERR_BAD_LEN
        assert (out[1] == 0).all()


def test_write_skips_negative_and_flags_out_of_range_slots():
    w = build("qwen", 8, batch=5, len_lo=1, len_hi=50)
    d = DeviceStep(w)
    slots = w.slot_mapping.copy()
    slots[1] = -1
    slots[3] = w.num_blocks * 16 + 7
    d.slots = torch.from_numpy(slots).cuda()
    d.write()
    assert d.err_word() & pkv.DEV_ERR_BAD_SLOT
    s2 = slots.copy()
    s2[3] = -1
    kc, vc = oracle.kv_write(w.k_cache, w.v_cache, w.k_new, w.v_new, s2)
    assert np.array_equal(host_bits(d.kc), kc) and np.array_equal(host_bits(d.vc), vc)


def test_python_binding_rejects_bad_tensors():
    w = build("tiny", 0)
    d = DeviceStep(w)
    with pytest.raises(TypeError):
        pkv.paged_kv_write(d.k_new.float(), d.v_new, d.kc, d.vc, d.slots)
    with pytest.raises(ValueError):
        pkv.paged_kv_write(d.k_new.cpu(), d.v_new, d.kc, d.vc, d.slots)
    with pytest.raises(ValueError):
        pkv.paged_attention_decode(d.out, d.q, d.kc, d.vc, d.tables[:2], d.lens, 0.1, 4)
    with pytest.raises(pkv.PkvError) as e:
        pkv.paged_attention_decode(d.out[:, :, :48].contiguous(), d.q[:, :, :48].contiguous(),
                                   d.kc[..., :48].contiguous(), d.vc[..., :48].contiguous(),
                                   d.tables, d.lens, 0.1, 4)
    assert e.value.code == pkv.ERR_UNSUPPORTED


def test_auto_split_edges():
    """Split-K through the automatic choice: a zero-length row, a bad table
    entry, lengths past the table or negative -- flagged, skipped, zero rows."""
    w = build("llama", 8, batch=9, len_lo=40, len_hi=700, head_dim=64)
    c = w.cfg
    assert pkv.decode_variant_for(c["batch"], c["num_heads"], c["num_kv_heads"], c["head_dim"],
                                  w.block_tables.shape[1], 512, 1 << 30) == pkv.DECODE_SPLIT
    d = DeviceStep(w)
    d.write()
    kc, vc = oracle.kv_write(w.k_cache, w.v_cache, w.k_new, w.v_new, w.slot_mapping)
    lens = w.lens.copy()
    lens[2] = 0
    ref = oracle.paged_decode(w.q, kc, vc, w.block_tables, lens, c["scale"])
    out = d.decode(pkv.DECODE_AUTO, 512, lens=torch.from_numpy(lens).cuda())
    assert (out[2] == 0).all()
    check_close(out, ref, "automatic split, zero-length row")
    assert d.err_word() == 0
    t = w.block_tables.copy()
    t[1, 1] = w.num_blocks + 7
    out = d.decode(pkv.DECODE_AUTO, 512, tables=torch.from_numpy(t).cuda())
    assert np.isfinite(bits_to_f64(out)).all()
    keep = [0] + list(range(2, c["batch"]))
    ref = oracle.paged_decode(w.q, kc, vc, w.block_tables, w.lens, c["scale"])
    check_close(out[keep], ref[keep], "automatic split, rows beside a bad table entry")
    assert d.err_word() & pkv.DEV_ERR_BAD_BLOCK
    d.err.zero_()
    lens = w.lens.copy()
    lens[0] = w.block_tables.shape[1] * 16 + 5
    lens[1] = -3
    out = d.decode(pkv.DECODE_AUTO, 512, lens=torch.from_numpy(lens).cuda())
    assert d.err_word() & pkv.DEV_ERR_BAD_LEN
    assert (out[1] == 0).all()


@pytest.mark.parametrize("variant,part", [(pkv.DECODE_AUTO, 512), (pkv.DECODE_SINGLE, 512),
                                          (pkv.DECODE_SPLIT, 64), (pkv.DECODE_CLUSTER, 128)])
def test_lengths_and_tables_written_by_the_kernel_just_before_the_call(variant, part):
    """The decode grids without a longest-first order read each sequence's
    length and table row before they wait for the kernel ahead of them on the
    stream.  A kernel that never lets dependents launch early (every torch
    kernel) may still write them right before the call.  Here torch kernels
    relabel two physical blocks (pool and tables) and then shorten the
    lengths, the last one immediately before the decode; the result is the
    oracle's for the shortened lengths (relabelling changes nothing)."""
    w = build("llama", 26, batch=6, len_lo=40, len_hi=700)
    kc, vc = oracle.kv_write(w.k_cache, w.v_cache, w.k_new, w.v_new, w.slot_mapping)
    cut = np.array([0, 5, 17, 1, 33, 2])
    lens2 = (np.asarray(w.lens) - cut).astype(np.int64)
    ref = oracle.paged_decode(w.q, kc, vc, w.block_tables, lens2, w.cfg["scale"])
    d = DeviceStep(w)
    d.write()
    a, b = int(w.block_tables[0, 0]), int(w.block_tables[1, 0])
    torch.cuda.synchronize()
    for cache in (d.kc, d.vc):
        tmp = cache[a].clone()
        cache[a] = cache[b]
        cache[b] = tmp
    ma, mb = d.tables == a, d.tables == b
    d.tables.masked_fill_(ma, b)
    d.tables.masked_fill_(mb, a)
    d.lens.sub_(torch.from_numpy(cut.astype(np.int32)).cuda())
    out = d.decode(variant, part)
    check_close(out, ref, f"metadata written just before the call, variant {variant}/{part}")
    assert d.err_word() == 0
