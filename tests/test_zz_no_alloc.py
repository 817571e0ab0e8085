"""pkv_paged_attention_decode_static: split-K decode for callers that must not
allocate device memory when they run (an engine plugin whose execution path
may not allocate, a server that reserves all memory at start-up, code that
avoids cudaMalloc/cudaFree because they can synchronise the device).  Its
scratch is a fixed array inside the library instead of a caller workspace.

Called through the C ABI on two calls in a row and compared with the regular
entry point (pkv_paged_attention_decode_ex, split-K, same partition, caller-
owned workspace): both run the same kernels on the same inputs, so the outputs
must be the same bits -- a stale or misaddressed scratch would shift them.
The output is also checked against the fp64 oracle with the tolerance of the
parity tests, and the device's free memory must not change across a call.
This file sorts last so that a failure here comes after every other test."""
import gc

import numpy as np
import pytest
import torch

from gpu_helpers import DeviceStep, build, check_close, host_bits, oracle_after_write

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


CASES = [("qwen", 21, dict(batch=6, len_lo=1, len_hi=1500), 512),
         ("llama", 22, dict(batch=5, len_lo=1, len_hi=900, head_dim=64), 64),
         ("long", 24, dict(batch=2, len_fixed=3000, num_blocks=420), 128)]


@pytest.mark.parametrize("name,seed,kw,part", CASES, ids=[c[0] for c in CASES])
def test_static_scratch_matches_regular_entry_twice_in_a_row(name, seed, kw, part):
    w = build(name, seed, **kw)
    d = DeviceStep(w)
    d.write()
    _, _, ref = oracle_after_write(w)
    rc, want = call_regular(d, part)
    assert rc == pkv.OK
    for call in range(2):  # the second call starts from the first call's scratch contents
        d.out.fill_(float("nan"))
        gc.collect()  # tensors freed late by the collector would show as a drop below
        torch.cuda.synchronize()
        free_before = torch.cuda.mem_get_info()[0]
        held_before = torch.cuda.memory_allocated()
        rc, got = call_static(d, part)
        assert rc == pkv.OK
        assert np.array_equal(got, want), f"call {call}: differs from the regular split-K entry"
        check_close(got, ref, f"static scratch {name}, call {call}")
        if call == 1:  # the first call may load the library's kernels; later calls take nothing
            assert torch.cuda.mem_get_info()[0] == free_before     # no cudaMalloc
            assert torch.cuda.memory_allocated() <= held_before    # nothing through torch
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
