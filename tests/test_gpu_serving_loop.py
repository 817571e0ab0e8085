"""An engine's life on one cache, step by step: new prompts (allocator
extend, the write kernel, tcgen05 prefill), decode steps over every live
sequence (batch append with copy-on-write copies, then the fused write +
decode), beams forked mid-block, sequences swapped out to pinned host memory
and back, sequences freed.  A host mirror of the cache and of the swap space
is updated only by the oracle's write / copy / swap; after every event the
GPU outputs are checked against the oracle's attention on the mirror, and
the whole pool and swap space are compared bit for bit along the way."""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import check_close, dev_bf16, host_bits

pytestmark = pytest.mark.gpu
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from paged_kv_cache_459_b200 import pkv  # noqa: E402
import workloads as wl  # noqa: E402

NB, NHOST = 192, 64


class Engine:
    def __init__(self, hq, hkv, d, seed):
        self.hq, self.hkv, self.d = hq, hkv, d
        self.scale = 1 / np.sqrt(d)
        self.rng = wl.rng(seed)
        self.seed = seed
        self.draws = 0
        self.alloc = pkv.BlockAllocator(NB, self.rng.permutation(NB))
        self.alloc.set_host_pool(NHOST)
        kc = wl.bf16_normal((NB, hkv, 16, d), seed, 0)
        vc = wl.bf16_normal((NB, hkv, 16, d), seed, 1)
        self.mk, self.mv = kc.copy(), vc.copy()                         # host mirror (oracle only)
        self.kc, self.vc = dev_bf16(kc), dev_bf16(vc)
        self.mhk = np.zeros((NHOST, hkv, 16, d), np.uint16)
        self.mhv = np.zeros_like(self.mhk)
        self.hk = torch.zeros((NHOST, hkv, 16, d), dtype=torch.bfloat16).pin_memory()
        self.hv = torch.zeros_like(self.hk).pin_memory()
        self.err = torch.zeros(1, dtype=torch.int32, device="cuda")
        self.live, self.swapped = set(), set()
        self.next_id = 0
        self.decodes = self.prefills = self.forks = self.swaps = self.frees = self.cows = 0

    def draw(self, shape):
        self.draws += 1
        return wl.bf16_normal(shape, self.seed + 1000, self.draws)

    # -------------------------------------------------------------- events
    def new_prompt(self, n):
        sid = self.next_id
        self.alloc.add_seq(sid, 0)
        try:
            slots = self.alloc.extend(sid, n)
        except pkv.AllocError:
            self.alloc.free_seq(sid)
            return
        self.next_id += 1
        k, v, q = self.draw((n, self.hkv, self.d)), self.draw((n, self.hkv, self.d)), self.draw((n, self.hq, self.d))
        pkv.paged_kv_write(dev_bf16(k), dev_bf16(v), self.kc, self.vc, torch.from_numpy(slots).cuda(), err=self.err)
        self.mk, self.mv = oracle.kv_write(self.mk, self.mv, k, v, slots)
        tables, lens = self.alloc.export([sid], -(-n // 16))
        qs = np.array([0, n], np.int32)
        out = torch.empty((n, self.hq, self.d), dtype=torch.bfloat16, device="cuda")
        pkv.paged_attention_prefill(out, dev_bf16(q), self.kc, self.vc, torch.from_numpy(tables).cuda(),
                                    torch.from_numpy(lens).cuda(), torch.from_numpy(qs).cuda(),
                                    self.scale, self.hkv, n, err=self.err)
        ref = oracle.paged_prefill(q, self.mk, self.mv, tables, lens, qs, self.scale)
        check_close(host_bits(out), ref, f"prefill of sequence {sid} ({n} tokens)")
        self.live.add(sid)
        self.prefills += 1

    def fork(self):
        cands = sorted(s for s in self.live - self.swapped if self.alloc.seq_len(s) > 0)
        if not cands:
            return
        parent = cands[int(self.rng.integers(len(cands)))]
        n = int(self.rng.integers(1, self.alloc.seq_len(parent) + 1))  # often mid-block
        child = self.next_id
        try:
            self.alloc.fork(parent, child, n)
        except pkv.AllocError:
            return
        self.next_id += 1
        self.live.add(child)
        self.forks += 1

    def swap_out(self):
        cands = sorted(self.live - self.swapped)
        if not cands:
            return
        s = cands[int(self.rng.integers(len(cands)))]
        try:
            self.alloc.swap_out(s)        # refused while the sequence holds shared blocks
        except pkv.AllocError:
            return
        self.move(pkv.SWAP_OUT)
        self.swapped.add(s)

    def swap_in(self):
        if not self.swapped:
            return
        s = sorted(self.swapped)[int(self.rng.integers(len(self.swapped)))]
        try:
            self.alloc.swap_in(s)
        except pkv.AllocError:
            return
        self.move(pkv.SWAP_IN)
        self.swapped.discard(s)

    def move(self, direction):
        g, h = self.alloc.take_swaps(direction)
        if len(g):
            pkv.swap_blocks(self.kc, self.vc, self.hk, self.hv, torch.from_numpy(g).cuda(),
                            torch.from_numpy(h).cuda(), direction, err=self.err)
            self.mk, self.mv, self.mhk, self.mhv = oracle.swap_blocks(
                self.mk, self.mv, self.mhk, self.mhv, g, h, 0 if direction == pkv.SWAP_OUT else 1)
        self.swaps += 1

    def free(self):
        if not self.live:
            return
        s = sorted(self.live)[int(self.rng.integers(len(self.live)))]
        self.alloc.free_seq(s)
        self.live.discard(s)
        self.swapped.discard(s)
        self.frees += 1

    def decode_step(self, variant, part):
        ids = sorted(self.live - self.swapped)
        if not ids:
            return
        try:
            slots = self.alloc.append_tokens(ids)
        except pkv.AllocError:
            self.free()                   # out of blocks: let the pool breathe
            return
        src, dst = self.alloc.take_copies()
        if len(src):                      # copy-on-write before the step's write
            pkv.copy_blocks(self.kc, self.vc, torch.from_numpy(src).cuda(), torch.from_numpy(dst).cuda(),
                            err=self.err)
            self.mk, self.mv = oracle.copy_blocks(self.mk, self.mv, src, dst)
            self.cows += len(src)
        width = max(-(-self.alloc.seq_len(s) // 16) for s in ids)
        tables, lens = self.alloc.export(ids, width)
        B = len(ids)
        q, k, v = self.draw((B, self.hq, self.d)), self.draw((B, self.hkv, self.d)), self.draw((B, self.hkv, self.d))
        out = torch.empty((B, self.hq, self.d), dtype=torch.bfloat16, device="cuda")
        pkv.paged_decode_step(out, dev_bf16(q), dev_bf16(k), dev_bf16(v), self.kc, self.vc,
                              torch.from_numpy(tables).cuda(), torch.from_numpy(lens).cuda(),
                              self.scale, self.hkv, variant=variant, partition_tokens=part, err=self.err)
        self.mk, self.mv = oracle.kv_write(self.mk, self.mv, k, v, slots)
        ref = oracle.paged_decode(q, self.mk, self.mv, tables, lens, self.scale)
        check_close(host_bits(out), ref, f"decode step {self.decodes} over {B} sequences")
        self.decodes += 1

    def check_pool(self, what):
        torch.cuda.synchronize()
        assert np.array_equal(host_bits(self.kc), self.mk), f"{what}: K pool differs"
        assert np.array_equal(host_bits(self.vc), self.mv), f"{what}: V pool differs"
        assert np.array_equal(host_bits(self.hk), self.mhk), f"{what}: host K differs"
        assert np.array_equal(host_bits(self.hv), self.mhv), f"{what}: host V differs"
        assert int(self.err.item()) == 0, f"{what}: device error word {int(self.err.item())}"


@pytest.mark.parametrize("hq,hkv,d,seed", [(8, 2, 64, 1), (4, 4, 128, 2)])
def test_serving_loop(hq, hkv, d, seed):
    e = Engine(hq, hkv, d, seed)
    for _ in range(3):
        e.new_prompt(int(e.rng.integers(1, 150)))
    variants = [(pkv.DECODE_AUTO, 512), (pkv.DECODE_SPLIT, 32), (pkv.DECODE_SINGLE, 512)]
    for step in range(48):
        r = float(e.rng.random())
        if r < 0.15 and len(e.live) < 9:
            e.new_prompt(int(e.rng.integers(1, 150)))
        elif r < 0.30:
            e.fork()
        elif r < 0.40:
            e.swap_out()
        elif r < 0.50:
            e.swap_in()
        elif r < 0.56 and len(e.live) > 2:
            e.free()
        e.decode_step(*variants[step % len(variants)])
        if step % 8 == 7:
            e.check_pool(f"step {step}")
    e.check_pool("end")
    # the loop has to have exercised every path
    assert e.decodes >= 40 and e.prefills >= 3 and e.forks >= 2 and e.cows >= 1 and e.swaps >= 2, \
        (e.decodes, e.prefills, e.forks, e.cows, e.swaps)
