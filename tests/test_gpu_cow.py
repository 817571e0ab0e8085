"""GPU parity of copy-on-write: beams forked mid-block share the parent's
blocks; each beam's next token makes the allocator queue a private copy of
the shared, partly filled block.  pkv_copy_blocks + write + decode must match
the oracle's copy + write + decode bit-exactly (caches) and within tolerance
(attention)."""
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


@pytest.mark.parametrize("hq,hkv,d,parent_len,beams", [(8, 8, 128, 1000, 4), (28, 4, 128, 77, 6),
                                                      (4, 4, 64, 33, 3)])
def test_beams_copy_on_write(hq, hkv, d, parent_len, beams):
    nb = 64 + 2 * beams + parent_len // 16
    gen = wl.rng(parent_len)
    bm = BlockManager(nb, gen.permutation(nb))
    bm.add_seq(0, parent_len)
    for b in range(1, beams):
        bm.fork(0, b)
    ids = list(range(beams))
    slots = np.array(bm.append_tokens(ids))
    src, dst = bm.take_copies()
    assert len(src) == (beams - 1 if parent_len % 16 else 0)
    kc = wl.bf16_normal((nb, hkv, 16, d), 1, 0)
    vc = wl.bf16_normal((nb, hkv, 16, d), 1, 1)
    k_new, v_new = wl.bf16_normal((beams, hkv, d), 1, 2), wl.bf16_normal((beams, hkv, d), 1, 3)
    q = wl.bf16_normal((beams, hq, d), 1, 4)
    tables, lens = bm.export(ids, (parent_len + 1 + 15) // 16)

    rk, rv = oracle.copy_blocks(kc, vc, src, dst)
    rk, rv = oracle.kv_write(rk, rv, k_new, v_new, slots)
    ref = oracle.paged_decode(q, rk, rv, tables, lens, 1 / np.sqrt(d))

    gk, gv = dev_bf16(kc), dev_bf16(vc)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkv.copy_blocks(gk, gv, torch.from_numpy(src).cuda(), torch.from_numpy(dst).cuda(), err=err)
    pkv.paged_kv_write(dev_bf16(k_new), dev_bf16(v_new), gk, gv, torch.from_numpy(slots).cuda(),
                       err=err)
    out = torch.empty((beams, hq, d), dtype=torch.bfloat16, device="cuda")
    pkv.paged_attention_decode(out, dev_bf16(q), gk, gv, torch.from_numpy(tables).cuda(),
                               torch.from_numpy(lens).cuda(), 1 / np.sqrt(d), hkv, err=err)
    torch.cuda.synchronize()
    assert np.array_equal(host_bits(gk), rk) and np.array_equal(host_bits(gv), rv)
    check_close(host_bits(out), ref, "beams after copy-on-write")
    assert int(err.item()) == 0


def test_copy_blocks_flags_bad_ids():
    kc = dev_bf16(wl.bf16_normal((8, 2, 16, 64), 2, 0))
    vc = dev_bf16(wl.bf16_normal((8, 2, 16, 64), 2, 1))
    before = host_bits(kc)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkv.copy_blocks(kc, vc, torch.tensor([0, 9, -1], device="cuda"),
                    torch.tensor([8, 1, 2], device="cuda"), err=err)
    torch.cuda.synchronize()
    assert int(err.item()) & pkv.DEV_ERR_BAD_BLOCK
    assert np.array_equal(host_bits(kc), before)
