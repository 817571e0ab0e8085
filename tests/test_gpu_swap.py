"""GPU parity of block swap (host swap space): sequences moved to pinned host
memory and back into other GPU blocks decode exactly as before; the host
copies match the oracle's bit for bit; a pointer the GPU cannot reach is an
argument error, not a fault."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import DeviceStep, build, host_bits

pytestmark = pytest.mark.gpu
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from paged_kv_cache_459_b200 import pkv  # noqa: E402
import workloads as wl  # noqa: E402


@pytest.mark.parametrize("name,kw", [("llama", dict(batch=6, len_lo=20, len_hi=300)),
                                     ("qwen", dict(batch=5, len_lo=20, len_hi=500))])
def test_swap_round_trip(name, kw):
    w = build(name, 8, pool_factor=2.0, **kw)
    d = DeviceStep(w)
    d.write()
    base = d.decode(pkv.DECODE_SINGLE)
    nhost = 128
    hk = torch.zeros((nhost,) + tuple(d.kc.shape[1:]), dtype=torch.bfloat16).pin_memory()
    hv = torch.zeros_like(hk).pin_memory()
    bm = w.alloc
    bm.set_host_pool(nhost)
    for s in (1, 4):
        bm.swap_out(s)
    g, h = bm.take_swaps(pkv.SWAP_OUT)
    pkv.swap_blocks(d.kc, d.vc, hk, hv, torch.from_numpy(g).cuda(), torch.from_numpy(h).cuda(),
                    pkv.SWAP_OUT, err=d.err)
    torch.cuda.synchronize()
    _, _, rhk, rhv = oracle.swap_blocks(host_bits(d.kc), host_bits(d.vc), host_bits(hk),
                                        host_bits(hv), g, h, 0)
    assert np.array_equal(host_bits(hk), rhk) and np.array_equal(host_bits(hv), rhv)
    d.kc[torch.from_numpy(g).cuda()] = float("nan")  # freed blocks get reused meanwhile
    d.vc[torch.from_numpy(g).cuda()] = float("nan")
    for s in (4, 1):
        bm.swap_in(s)
    g2, h2 = bm.take_swaps(pkv.SWAP_IN)
    pkv.swap_blocks(d.kc, d.vc, hk, hv, torch.from_numpy(g2).cuda(), torch.from_numpy(h2).cuda(),
                    pkv.SWAP_IN, err=d.err)
    tables, lens = bm.export(list(range(w.cfg["batch"])), w.block_tables.shape[1])
    assert not np.array_equal(tables, w.block_tables)
    out = d.decode(pkv.DECODE_SINGLE, tables=torch.from_numpy(tables).cuda())
    assert np.array_equal(out, base)
    assert d.err_word() == 0


def test_swap_rejects_unpinned_host_memory():
    w = build("tiny", 0)
    d = DeviceStep(w)
    host = np.zeros((4,) + tuple(d.kc.shape[1:]), np.uint16)  # pageable, not registered
    ids = torch.zeros(1, dtype=torch.int64, device="cuda")
    rc = pkv.lib().pkv_swap_blocks(d.kc.data_ptr(), d.vc.data_ptr(), host.ctypes.data,
                                   host.ctypes.data, ids.data_ptr(), ids.data_ptr(), 1,
                                   pkv.SWAP_OUT, 4, 64, w.num_blocks, 4, None,
                                   torch.cuda.current_stream().cuda_stream)
    assert rc == pkv.ERR_INVALID_ARG
    with pytest.raises(ValueError):
        pkv.swap_blocks(d.kc, d.vc, torch.zeros(4, 4, 16, 64, dtype=torch.bfloat16),
                        torch.zeros(4, 4, 16, 64, dtype=torch.bfloat16), ids, ids, pkv.SWAP_OUT)
