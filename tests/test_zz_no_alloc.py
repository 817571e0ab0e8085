"""pkv_paged_attention_decode_static: split-K decode for callers that must not
allocate device memory when they run (an engine plugin whose execution path
may not allocate, a server that reserves all memory at start-up, code that
avoids cudaMalloc/cudaFree because they can synchronise the device).  Its
scratch is a fixed array inside the library instead of a caller workspace.

Called through the C ABI and compared with the regular entry point
(pkv_paged_attention_decode_ex, split-K, caller-owned workspace) on the same
inputs, two calls in a row, with the tolerance of the parity tests.  This file
sorts last so that a failure here comes after every other test has run."""
import numpy as np
import pytest
import torch

from gpu_helpers import ATOL, RTOL, DeviceStep, bits_to_f64, build, host_bits

pytestmark = pytest.mark.gpu
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from paged_kv_cache_459_b200 import pkv  # noqa: E402

LIMIT = 32 << 20  # PKV_STATIC_SCRATCH_BYTES


def _args(d: DeviceStep, partition):
    w = d.w
    c = w.cfg
    return (d.out.data_ptr(), d.q.data_ptr(), d.kc.data_ptr(), d.vc.data_ptr(),
            d.tables.data_ptr(), d.tables.shape[1], d.lens.data_ptr(), c["batch"],
            c["num_heads"], c["num_kv_heads"], c["head_dim"], w.num_blocks, c["scale"], partition)


def call_static(d: DeviceStep, partition=512):
    stream = torch.cuda.current_stream().cuda_stream
    rc = pkv.lib().pkv_paged_attention_decode_static(*_args(d, partition), d.err.data_ptr(), stream)
    torch.cuda.synchronize()
    return rc, host_bits(d.out)


def call_regular(d: DeviceStep, partition=512):
    c = d.w.cfg
    need = pkv.decode_workspace_bytes(c["batch"], c["num_heads"], c["head_dim"],
                                      d.tables.shape[1], partition)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    a = _args(d, partition)
    rc = pkv.lib().pkv_paged_attention_decode_ex(*a[:13], pkv.DECODE_SPLIT, partition,
                                                 ws.data_ptr(), need, d.err.data_ptr(), stream)
    torch.cuda.synchronize()
    return rc, host_bits(d.out)


def assert_match(got_bits, want_bits):
    got, want = bits_to_f64(got_bits), bits_to_f64(want_bits)
    assert np.isfinite(got).all() and np.isfinite(want).all()
    assert np.all(np.abs(got - want) <= ATOL + RTOL * np.abs(want))


def test_static_scratch_matches_regular_entry_twice_in_a_row():
    cases = [build("qwen", 21, batch=6, len_lo=1, len_hi=1500),
             build("llama", 22, batch=5, len_lo=1, len_hi=900, head_dim=64)]
    steps = [DeviceStep(w) for w in cases]
    for d in steps:
        d.write()
    for d, part in ((steps[0], 512), (steps[1], 64)):
        rc, want = call_regular(d, part)
        assert rc == pkv.OK
        for _ in range(2):  # the second call starts from the first call's scratch contents
            d.out.fill_(float("nan"))
            rc, got = call_static(d, part)
            assert rc == pkv.OK
            assert_match(got, want)
        assert d.err_word() == 0


def test_static_scratch_rejects_sizes_past_its_limit():
    w = build("qwen", 23, batch=4, len_lo=1, len_hi=64)
    d = DeviceStep(w)
    c = w.cfg
    # a table so wide that the split-K partials need more than the fixed array
    width = LIMIT // (c["batch"] * c["num_heads"] * (c["head_dim"] + 2) * 4) * 32 + 64
    assert pkv.decode_workspace_bytes(c["batch"], c["num_heads"], c["head_dim"], width, 512) > LIMIT
    wide = torch.full((c["batch"], width), -1, dtype=torch.int32, device="cuda")
    wide[:, : d.tables.shape[1]] = d.tables
    d.tables = wide
    rc, _ = call_static(d)
    assert rc == pkv.ERR_WORKSPACE
