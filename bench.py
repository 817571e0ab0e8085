#!/usr/bin/env python
"""Benchmark of the paged KV-cache decode step on B200.

One step = the whole hot path over one batch: the cache write of every
sequence's new token and single-query decode attention over the paged cache,
in one library call (pkv_paged_decode_step; the write fused into the decode
kernel).  Block tables and slots come from the library's C++ block
allocator; values are seeded synthetic bf16 N(0,1) draws.  Prints ONE JSON
line (rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config qwen]
    python bench.py --impl reference ...     # the fp64 CPU oracle, timed on host cores
    python bench.py --row prefill|cow|swap|alloc   # the rows beside the decode step

The headline workload is the Qwen2.5-7B-shaped GQA decode (batch 256, 28/4
heads).  At N = 1 the same line also carries the Llama-2-7B-shaped and the
long-context (8 x 32768, split-K) workloads, the shared-prefix cascade, a
batch sweep and the paged prefill, each with its own roofline and clocks
(--no-extras leaves them out).

Multi-GPU (torchrun, one process per GPU): every rank decodes its own batch
(seed + rank) -- independent problems, no collective on the data path -- and
the job time is the max over ranks of the device-timed K steps.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "paged decode attention: KV HBM GB/s (% of B200 peak) and sequences·steps/sec"
UNIT = "seq*steps/s"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126 * 1024 * 1024

WORKLOAD_NAMES = {
    "tiny": "tiny paged decode: 4 seqs, lens {1,17,33,100}, 4/4 heads, d 64",
    "llama": "Llama-2-7B-shaped MHA decode: batch 64, 32/32 heads, d 128, len U[128,2048]",
    "qwen": "Qwen2.5-7B-shaped GQA decode: batch 256, 28/4 heads, d 128, len U[512,4096]",
    "prefix": "prefix-shared decode: batch 128, 2000-token shared prefix + U[16,512], 32/32, d 128",
    "long": "long-context GQA decode: batch 8 x 32768, 32/8 heads, d 128, 512-token split-K",
}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["pkv", "reference"], default="pkv")
    ap.add_argument("--config", choices=sorted(WORKLOAD_NAMES), default="qwen")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--batch", type=int, default=None,
                    help="override the workload's batch (smaller cases for ncu captures)")
    ap.add_argument("--variant", choices=["auto", "single", "split", "cluster"], default="auto")
    ap.add_argument("--partition", type=int, default=512)
    ap.add_argument("--row", choices=["decode", "prefill", "cow", "swap", "alloc"], default="decode",
                    help="which part of the path to measure (decode: the default step)")
    ap.add_argument("--cascade", action="store_true",
                    help="shared-prefix decode: prefix blocks read once per group and KV head")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--unfused", action="store_true",
                    help="time the step as separate write and decode calls (the default step "
                         "is pkv_paged_decode_step, the write fused into the decode kernel)")
    ap.add_argument("--flush-l2", action="store_true",
                    help="write a 256 MB buffer between timed steps (automatic when the "
                         "step's K/V fit in L2) and time the step from per-step events")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="CPU time budget of the oracle baseline sample")
    ap.add_argument("--no-extras", action="store_true",
                    help="only the headline workload (no llama / long / cascade keys, batch "
                         "sweep or prefill; these run by default at N = 1)")
    return ap.parse_args()


def measured_peak_hbm():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def algorithmic_bytes(w) -> dict:
    """Bytes the decode step must move at minimum: every sequence's K and V
    rows once (len x Hkv x d x 2 B, twice) plus Q; the write moves the new
    K/V rows in and out."""
    cfg = w.cfg
    d, hq, hkv = cfg["head_dim"], cfg["num_heads"], cfg["num_kv_heads"]
    toks = int(np.asarray(w.lens, dtype=np.int64).sum())
    kv = toks * hkv * d * 2 * 2
    q = cfg["batch"] * hq * d * 2
    out = cfg["batch"] * hq * d * 2
    write = cfg["batch"] * hkv * d * 2 * 2 * 2
    return dict(kv=kv, q=q, out=out, write=write, tokens=toks)


def max_over_ranks(values, device=None):
    """Element-wise max of a list of floats over all ranks (identity when not
    distributed): the job time is the slowest rank's."""
    import torch
    import torch.distributed as dist

    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.cpu()]


def job_throughput(units_per_rank: int, steps: int, world: int, job_ms: float) -> float:
    """Units all ranks processed per second of the slowest rank's time."""
    return units_per_rank * steps * world / (job_ms * 1e-3)


def source_sha(*paths: str) -> str:
    h = hashlib.sha1()
    for path in paths:
        with open(path, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:12]


def committed_traffic(kernel: str, workload: str):
    """dram read+write bytes per launch from the committed ncu summary, if it
    was taken on the current source of the kernel (the file named in the
    record, by its sha1 prefix)."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            rec = json.load(f)[workload][kernel]
    except (OSError, KeyError, ValueError):
        return None
    names = rec.get("source", [])
    paths = [os.path.join(ROOT, "paged_kv_cache_459_b200", "csrc", n)
             for n in ([names] if isinstance(names, str) else names)]
    if not paths or not all(os.path.isfile(x) for x in paths) or \
            rec.get("source_sha") != source_sha(*paths):
        return None
    return rec.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the GPU is loaded."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_id: str | None):
        self.proc = None
        self.lines: list[str] = []
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
               "-lms", "50"]
        if device_id:
            cmd += ["--id", device_id]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
        except OSError:
            self.proc = None

    def stop(self) -> dict | None:
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = [r.split(",") for r in out.strip().splitlines() if r.count(",") >= 8]
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if "Active" in v
                          and "Not" not in v})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(rows)}


def device_pci_id(dev) -> str | None:
    import torch
    try:
        p = torch.cuda.get_device_properties(dev)
        return f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
    except Exception:
        return None


# ----------------------------------------------------------------- CPU oracle
class OracleStep:
    """The fp64 oracle as it stands (C, OpenMP over sequence x KV head) run as
    one decode step -- write + decode, in place -- over the first `nseq`
    sequences of a workload, on the host cores."""

    def __init__(self, w):
        import oracle
        self.lib = oracle.lib()
        self.cores = oracle.threads_available()
        self.threads = self.cores
        self.w = w
        self.kc, self.vc = w.k_cache.copy(), w.v_cache.copy()
        c = w.cfg
        self.out = np.zeros((c["batch"], c["num_heads"], c["head_dim"]), np.float64)
        self.tables = np.ascontiguousarray(w.block_tables, np.int32)
        self.lens = np.ascontiguousarray(w.lens, np.int32)

    def __call__(self, nseq: int) -> None:
        w, c = self.w, self.w.cfg
        self.lib.oracle_kv_write(self.kc.ctypes.data, self.vc.ctypes.data, w.k_new.ctypes.data,
                                 w.v_new.ctypes.data, w.slot_mapping.ctypes.data, nseq,
                                 c["num_kv_heads"], c["head_dim"], w.num_blocks)
        rc = self.lib.oracle_paged_decode(
            self.out.ctypes.data, w.q.ctypes.data, self.kc.ctypes.data, self.vc.ctypes.data,
            self.tables.ctypes.data, self.tables.shape[1], self.lens.ctypes.data, nseq,
            c["num_heads"], c["num_kv_heads"], c["head_dim"], w.num_blocks, float(c["scale"]),
            self.threads)
        if rc != 0:
            raise RuntimeError(f"oracle failed ({rc})")

    def seconds_per_seq(self) -> float:
        n = min(4, self.w.cfg["batch"])
        t0 = time.perf_counter()
        self(n)
        return max(time.perf_counter() - t0, 1e-5) / n

    def timed(self, nseq: int, reps: int) -> float:
        t0 = time.perf_counter()
        for _ in range(reps):
            self(nseq)
        return time.perf_counter() - t0


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_baseline(w, budget_s: float) -> dict:
    """Bounded sample of the oracle on this host: about `budget_s` seconds on
    all the process's cores, then about a quarter of that on one thread."""
    st = OracleStep(w)
    st.seconds_per_seq()  # the first call pays page faults and cold caches
    per_seq = st.seconds_per_seq()
    b = w.cfg["batch"]
    nseq = int(min(b, max(1, budget_s / 3 / per_seq)))
    reps = max(1, int(budget_s / (nseq * per_seq)))
    el = st.timed(nseq, reps)
    st.threads = 1
    per_seq1 = st.seconds_per_seq()
    nseq1 = int(min(b, max(1, budget_s / 4 / per_seq1)))
    el1 = st.timed(nseq1, 1)
    return {"value": nseq * reps / el, "unit": UNIT, "cores": st.cores, "kind": "oracle",
            "sample": f"{reps} oracle steps (KV write + decode, fp64) over the first {nseq} of "
                      f"{b} sequences, {el:.1f} s on {st.cores} threads",
            "single_thread": {"value": nseq1 / el1, "unit": UNIT,
                              "sample": f"1 step over the first {nseq1} sequences, {el1:.1f} s"},
            "cpu_model": cpu_model()}


def run_reference(args):
    if int(os.environ.get("RANK", "0")) != 0:
        return 0
    from oracle.alloc_model import BlockManager
    import workloads as wl
    w = wl.build(args.config, args.seed, BlockManager)
    st = OracleStep(w)
    per_seq = st.seconds_per_seq()
    b = w.cfg["batch"]
    per_step = 120.0 / max(1, args.steps + args.warmup)  # the whole run within ~2 minutes
    nseq = int(min(b, max(1, per_step / per_seq)))
    st.timed(nseq, args.warmup)
    el = st.timed(nseq, args.steps)
    val = nseq * args.steps / el
    line = {
        "metric": METRIC, "value": val, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1000.0 * el / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD_NAMES[args.config], "name": args.config,
                   "sample_seqs_per_step": nseq},
        "impl": "reference",
        "cpu_baseline": {"value": val, "unit": UNIT, "cores": st.cores, "kind": "oracle",
                         "sample": f"each step: oracle KV write + decode (fp64) over the first "
                                   f"{nseq} of {b} sequences"},
        "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------- GPU path
# The host keeps ahead of the device in every timed loop: a spin kernel
# (torch.cuda._sleep) holds the stream while the first steps are enqueued, so
# the per-step events see the step's own device time rather than gaps left by
# the host issuing launches.  Spins sit outside the per-step events.
SPIN_CYCLES_LEAD = 20_000_000   # ~10 ms at the B200's clocks
SPIN_CYCLES_CHUNK = 4_000_000   # ~2 ms, before every FLUSH_CHUNK flushed steps
FLUSH_CHUNK = 16


class Resident:
    """One decode workload resident on the GPU (caches, step inputs, tables,
    workspace) with the step's library calls bound to it."""

    def __init__(self, args, name: str, seed: int, dev, *, batch=None, cascade=False,
                 variant="auto", partition=512, host_copies=False):
        import torch

        from paged_kv_cache_459_b200 import pkv
        import workloads as wl

        self.pkv, self.dev, self.name, self.cascade = pkv, dev, name, cascade
        self.partition = partition
        w = self.w = wl.build(name, seed, pkv.BlockAllocator, batch=batch)
        cfg = w.cfg
        self.B, self.hq, self.hkv, self.d = cfg["batch"], cfg["num_heads"], cfg["num_kv_heads"], cfg["head_dim"]
        self.scale = cfg["scale"]

        def up(bits):
            return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)

        q_h, k_h, v_h = (up(x) for x in (w.q, w.k_new, w.v_new))
        tables_h = torch.from_numpy(w.block_tables)
        lens_h = torch.from_numpy(w.lens.astype(np.int32))
        slots_h = torch.from_numpy(w.slot_mapping)
        if host_copies:  # pinned host inputs of the end-to-end loop
            q_h, k_h, v_h, tables_h, lens_h, slots_h = (
                t.pin_memory() for t in (q_h, k_h, v_h, tables_h, lens_h, slots_h))
            self.host = {"q": q_h, "k": k_h, "v": v_h, "tables": tables_h, "lens": lens_h,
                         "slots": slots_h}
        self.kc = up(w.k_cache).to(dev)
        self.vc = up(w.v_cache).to(dev)
        if not host_copies:  # the device holds them now
            w.k_cache = w.v_cache = None
        self.q, self.k_new, self.v_new = q_h.to(dev), k_h.to(dev), v_h.to(dev)
        self.tables, self.lens, self.slots = tables_h.to(dev), lens_h.to(dev), slots_h.to(dev)
        self.out = torch.empty_like(self.q)
        self.err = torch.zeros(1, dtype=torch.int32, device=dev)
        self.variant = {"auto": pkv.DECODE_AUTO, "single": pkv.DECODE_SINGLE,
                        "split": pkv.DECODE_SPLIT, "cluster": pkv.DECODE_CLUSTER}[variant]
        W = self.W = w.block_tables.shape[1]
        if cascade:
            pb_h, offs_h, mem_h = w.alloc.prefix_groups(list(range(self.B)))
            self.pb_h, self.offs_h, self.mem_h = pb_h, offs_h, mem_h
            self.pb, self.offs_g, self.mem = (torch.from_numpy(x).to(dev) for x in (pb_h, offs_h, mem_h))
            self.suffix_bound = pkv.suffix_blocks_bound(w.lens, pb_h)  # the allocator's host view
            ws_bytes = pkv.decode_prefix_workspace_bytes(self.B, self.hq, self.d, W, partition)
        else:
            ws_bytes = pkv.decode_workspace_bytes_for(self.variant, self.B, self.hq, self.hkv,
                                                      self.d, W, partition)
        self.ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
        self.chosen = self.variant if self.variant != pkv.DECODE_AUTO else pkv.decode_variant_for(
            self.B, self.hq, self.hkv, self.d, W, partition, self.ws.numel())
        self.parts = pkv.decode_cluster_parts_for(self.B, self.hq, self.hkv, self.d, W, self.variant,
                                                  partition, self.ws.numel()) if not cascade else 0

        self.fused = not args.unfused

    # -- the library calls of one step
    def write(self, c=None, o=None):
        c = c or {"k": self.k_new, "v": self.v_new, "slots": self.slots}
        self.pkv.paged_kv_write(c["k"], c["v"], self.kc, self.vc, c["slots"], err=self.err)

    def decode(self, c=None, o=None):
        c = c or {"q": self.q, "tables": self.tables, "lens": self.lens}
        o = self.out if o is None else o
        if self.cascade:
            self.pkv.paged_attention_decode_prefix(
                o, c["q"], self.kc, self.vc, c["tables"], c["lens"], self.scale, self.hkv, self.pb,
                self.offs_g, self.mem, max_suffix_blocks=self.suffix_bound,
                partition_tokens=self.partition, workspace=self.ws, err=self.err)
        else:
            self.pkv.paged_attention_decode(o, c["q"], self.kc, self.vc, c["tables"], c["lens"],
                                            self.scale, self.hkv, variant=self.variant,
                                            partition_tokens=self.partition, workspace=self.ws,
                                            err=self.err)

    def fused_step(self, c=None, o=None):
        """The write of each sequence's new token fused into the decode kernel."""
        c = c or {"q": self.q, "k": self.k_new, "v": self.v_new, "tables": self.tables,
                  "lens": self.lens}
        o = self.out if o is None else o
        if self.cascade:
            self.pkv.paged_decode_prefix_step(
                o, c["q"], c["k"], c["v"], self.kc, self.vc, c["tables"], c["lens"], self.scale,
                self.hkv, self.pb, self.offs_g, self.mem, max_suffix_blocks=self.suffix_bound,
                partition_tokens=self.partition, workspace=self.ws, err=self.err)
        else:
            self.pkv.paged_decode_step(o, c["q"], c["k"], c["v"], self.kc, self.vc, c["tables"],
                                       c["lens"], self.scale, self.hkv, variant=self.variant,
                                       partition_tokens=self.partition, workspace=self.ws,
                                       err=self.err)

    def add_cache_copies(self, n: int):
        """n more copies of the K/V pool -- the caches of a model's other layers:
        steps that rotate over them find none of their K/V in L2."""
        self.caches = [(self.kc, self.vc)] + [(self.kc.clone(), self.vc.clone()) for _ in range(n)]
        self.cur = 0

    def next_cache(self):
        self.cur = (self.cur + 1) % len(self.caches)
        self.kc, self.vc = self.caches[self.cur]

    def drop_cache_copies(self):
        self.kc, self.vc = self.caches[0]
        self.caches, self.cur = [(self.kc, self.vc)], 0

    def step(self, c=None, o=None):
        if self.fused:
            self.fused_step(c, o)
        else:
            self.write(c, o)
            self.decode(c, o)

    def two_calls(self):
        self.write()
        self.decode()

    # -- accounting
    def bytes(self) -> dict:
        ab = algorithmic_bytes(self.w)
        dec = ab["kv"] + ab["q"]
        if self.cascade:
            # what the cascade must read: each group's prefix once, every suffix once
            w = self.w
            uniq = int((np.asarray(w.lens, np.int64) - 16 * self.pb_h.astype(np.int64)).sum())
            uniq += sum(16 * int(self.pb_h[self.mem_h[self.offs_h[g]]])
                        for g in range(len(self.offs_h) - 1))
            dec = uniq * self.hkv * self.d * 2 * 2 + ab["q"]
        if self.fused:  # the new tokens' K/V: read once, written once
            dec += 2 * self.B * self.hkv * self.d * 2 * 2
        ab["decode"] = dec
        return ab

    def ordered(self) -> bool:
        """Whether the decode runs its sequences longest first (an order kernel)."""
        if self.cascade:
            return False
        if self.chosen == self.pkv.DECODE_CLUSTER:
            return self.B >= 16 and self.ws.numel() >= (4 * self.B + 255) // 256 * 256
        return self.chosen == self.pkv.DECODE_SINGLE and self.ws.numel() >= 4 * self.B

    def launches_per_step(self) -> int:
        pkv = self.pkv
        if self.cascade:  # (write;) prefix spans + suffix split-K in one launch, merge
            return 2 if self.fused else 3
        return (1 if self.fused else 2) + (1 if self.chosen == pkv.DECODE_SPLIT else 0) + \
            (1 if self.ordered() else 0)

    def variant_text(self) -> str:
        pkv = self.pkv
        if self.cascade:
            return "shared-prefix cascade (prefix once per group x KV head, split-K suffixes, merge)"
        return {pkv.DECODE_SINGLE: "single pass (one CTA per sequence x KV head, longest first)"
                if self.ordered() else "single pass (one CTA per sequence x KV head)",
                pkv.DECODE_SPLIT: "split-K %d-token partitions + merge" % self.partition,
                pkv.DECODE_CLUSTER: f"cluster split ({self.parts} equal parts per sequence, one "
                                    f"CTA each, merged in distributed shared memory" +
                                    (", longest first)" if self.ordered() else ")"),
                }[self.chosen]

    def kernel_text(self) -> str:
        pkv = self.pkv
        if self.cascade:
            return ("cascade_kernel (prefix spans + suffix units" +
                    (", fused write" if self.fused else "") + ") + cascade_merge_kernel")
        return (("paged_decode_kernel with the fused write" if self.fused else "paged_decode_kernel")
                + (" (cluster mode)" if self.chosen == pkv.DECODE_CLUSTER else "")
                + (" + merge kernel" if self.chosen == pkv.DECODE_SPLIT else "")
                + (" + order kernel" if self.ordered() else ""))

    def check_err(self, when: str):
        import torch
        torch.cuda.synchronize(self.dev)
        if int(self.err.item()) != 0:
            raise SystemExit(f"{self.name}: device error word {int(self.err.item())} {when}")


class L2Flush:
    """Empties L2 between timed steps: a 256 MB buffer is written (L2 then
    holds none of the step's inputs), then another 256 MB is read, so that the
    dirty lines of that write go back to HBM here rather than inside the next
    step (whose misses would otherwise pay for their write-back)."""

    def __init__(self, dev):
        import torch
        self.w = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)
        self.r = torch.zeros(2 * L2_BYTES // 4, dtype=torch.int32, device=dev)

    def __call__(self):
        self.w.zero_()
        self.r.sum()


def device_steps(step, K: int, dev, flush_buf=None):
    """Device time of K calls of step(): per-step times (ms each) and the
    whole loop (ms).  Without flush_buf the K steps run back to back between
    two events and each step is the loop's mean; with flush_buf (an L2Flush),
    L2 is emptied before every step, outside that step's own two events."""
    import torch

    stream = torch.cuda.current_stream(dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(K)] if flush_buf is not None else []
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    torch.cuda._sleep(SPIN_CYCLES_LEAD)
    t0.record(stream)
    for i in range(K):
        if flush_buf is not None:
            if i and i % FLUSH_CHUNK == 0:
                torch.cuda._sleep(SPIN_CYCLES_CHUNK)
            flush_buf()  # L2 holds none of this step's inputs and no dirty lines
            ev[i][0].record(stream)
        step()
        if flush_buf is not None:
            ev[i][1].record(stream)
    t1.record(stream)
    torch.cuda.synchronize(dev)
    loop = t0.elapsed_time(t1)
    if flush_buf is None:
        return [loop / K] * K, loop
    return [a.elapsed_time(b) for a, b in ev], loop


def rotating_steps(r: Resident, K: int, dev, fn=None) -> float:
    """Device time (ms) of K steps (fn, default r.step) back to back, each on
    the next copy of the K/V pool (Resident.add_cache_copies)."""
    import torch

    fn = fn or r.step
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    torch.cuda._sleep(SPIN_CYCLES_LEAD)
    t0.record()
    for _ in range(K):
        r.next_cache()
        fn()
    t1.record()
    torch.cuda.synchronize(dev)
    return t0.elapsed_time(t1)


def timed_decode(r: Resident, K: int, W: int, *, world: int, sampler=None, flush=None) -> dict:
    """W warm-up steps, then K timed steps of the resident workload; returns the
    line's numbers for it (and its clocks when a sampler runs).

    A workload whose K/V fits in L2 is timed two ways.  Rotating (the step
    time reported): the pool is copied until the copies hold over 3 L2 sizes
    and each step runs on the next copy, K steps back to back between two
    events -- as in a model, whose layers each read their own cache, so that a
    step's K/V were last touched two L2 sizes of traffic ago.  Flushed
    (reported beside it): L2 emptied before every step and each step timed
    alone by its own events, which adds the launch and event overhead of an
    isolated kernel (about 5 us on a B200 for an empty kernel)."""
    import torch

    for _ in range(W):
        r.step()
        if r.fused:
            r.two_calls()
    r.check_err("after warm-up")
    ab = r.bytes()
    if flush is None:  # the same choice on every rank
        flush = max_over_ranks([float(ab["kv"])], device=r.dev)[0] <= L2_BYTES
    flush_buf = L2Flush(r.dev) if flush else None
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    per, loop_ms = device_steps(r.step, K, r.dev, flush_buf)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    total_ms = sum(per) if flush else loop_ms  # the flushes are not the step's work
    flushed_us, copies = None, 1
    if flush:
        del flush_buf
        pool = 2 * r.kc.numel() * r.kc.element_size()
        copies = max(2, -(-3 * L2_BYTES // max(ab["kv"], 1)))
        free = torch.cuda.mem_get_info(r.dev)[0]
        copies = int(min(copies, 1 + (free // 2) // max(pool, 1)))
        r.add_cache_copies(copies - 1)
        for _ in range(2 * copies):  # every copy written and read once
            r.next_cache()
            r.step()
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
        loop_ms = rotating_steps(r, K, r.dev)
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
        r.drop_cache_copies()
        flushed_us = 1e3 * statistics.fmean(per)
        per = [loop_ms / K] * K
        total_ms = loop_ms
    clocks = None
    if sampler is not None:  # keep the GPU loaded long enough for the sampler to see it
        t0 = time.perf_counter()
        while time.perf_counter() - t0 < 1.0:
            for _ in range(50):
                r.step()
            torch.cuda.synchronize(r.dev)
        clocks = sampler.stop()
    r.check_err("after the timed steps")
    total_ms = max_over_ranks([total_ms], device=r.dev)[0]
    step_us = 1e3 * statistics.fmean(per)
    peak, peak_kind = measured_peak_hbm()
    achieved = ab["decode"] / (step_us * 1e-6) / 1e9
    return {
        "step_us": step_us, "total_ms": total_ms, "flush": flush, "bytes": ab,
        "flushed_step_us": flushed_us, "cache_copies": copies,
        "flushed_frac_of_measured_copy": None if flushed_us is None else
        ab["decode"] / (flushed_us * 1e-6) / 1e9 / peak,
        "value": job_throughput(r.B, K, world, total_ms),
        "kv_hbm_gbs": achieved,
        "kv_frac_of_8tbs": achieved / NOMINAL_HBM_GBS,
        "kv_frac_of_measured_copy": achieved / peak,
        "roofline": {
            "bound": "hbm", "kernel": r.kernel_text(),
            "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
            "peak_kind": peak_kind,
            "traffic": committed_traffic("cascade_kernel" if r.cascade else "paged_decode_kernel",
                                         ("prefix_cascade" if r.cascade else r.name)
                                         if r.B == CONFIG_BATCH.get(r.name) else None),
            "algorithmic_bytes_per_launch": ab["decode"],
        },
        "clocks": clocks,
    }


CONFIG_BATCH = {"tiny": 4, "llama": 64, "qwen": 256, "prefix": 128, "long": 8}


def workload_key(args, name, *, dev, cascade=False, batch=None, clocks=True) -> dict:
    """One extra workload of the bench line: the fused step timed like the
    headline, its roofline against the measured copy rate, and its clocks."""
    import torch

    r = Resident(args, name, args.seed, dev, batch=batch, cascade=cascade)
    sampler = ClockSampler(device_pci_id(dev)) if clocks else None
    m = timed_decode(r, args.steps, max(3, args.warmup), world=1, sampler=sampler)
    out = {
        "workload": WORKLOAD_NAMES[name] if batch is None else
        f"{WORKLOAD_NAMES[name]} (batch {r.B})",
        "variant": r.variant_text(), "step": "fused write + decode (one call)" if r.fused else
        "write, then decode", "tokens": m["bytes"]["tokens"],
        "decode_us": m["step_us"], "value": m["value"], "unit": UNIT,
        "kv_hbm_gbs": m["kv_hbm_gbs"], "kv_frac_of_8tbs": m["kv_frac_of_8tbs"],
        "kv_frac_of_measured_copy": m["kv_frac_of_measured_copy"],
        "l2": (f"inputs smaller than L2: each step on the next of {m['cache_copies']} copies of "
               f"the K/V pool (over 3 L2 sizes, as a model's layers), K steps back to back")
        if m["flush"] else "inputs larger than L2, no flush",
        "roofline": m["roofline"], "gpu_launches": args.steps * r.launches_per_step(),
    }
    if m["flush"]:
        out["flushed"] = flushed_key(m)
    if clocks:
        out["clocks"] = m["clocks"]
    if cascade:
        out["logical_kv_bytes"] = m["bytes"]["kv"]
        out["unique_kv_bytes"] = m["bytes"]["decode"] - m["bytes"]["q"] - \
            (2 * r.B * r.hkv * r.d * 2 * 2 if r.fused else 0)
    del r
    torch.cuda.empty_cache()
    return out


def flushed_key(m: dict) -> dict:
    """The same step timed alone: L2 flushed before it, its own two events."""
    return {"step_us": m["flushed_step_us"],
            "kv_frac_of_measured_copy": m["flushed_frac_of_measured_copy"],
            "how": "L2 flushed before every step (256 MB write, then 256 MB read), each step "
                   "between its own two events; an empty kernel measures ~5 us this way"}


def batch_sweep_key(args, dev) -> dict:
    """Llama-2-7B-shaped decode at batch 1 .. 128 (the pages' own batch sweep
    runs 1, 8, 32, 64, 128): small batches are latency-bound, large ones read
    at the copy rate."""
    import torch

    rows = []
    sampler = ClockSampler(device_pci_id(dev))
    # at least 200 timed steps per row: a batch-1 step is ~11 us, so that K = 20 would
    # time ~0.2 ms in all
    steps = max(args.steps, 200)
    for B in (1, 8, 32, 64, 128):
        r = Resident(args, "llama", args.seed, dev, batch=B)
        m = timed_decode(r, steps, max(3, args.warmup), world=1)
        row = {"batch": B, "steps": steps, "variant": r.variant_text(), "decode_us": m["step_us"],
               "kv_hbm_gbs": m["kv_hbm_gbs"],
               "kv_frac_of_measured_copy": m["kv_frac_of_measured_copy"],
               "value": m["value"],
               "l2": f"rotating over {m['cache_copies']} pool copies" if m["flush"] else
               "larger than L2",
               "algorithmic_bytes_per_launch": m["bytes"]["decode"]}
        if m["flush"]:
            row["flushed"] = flushed_key(m)
        rows.append(row)
        last = r
        if B != 128:
            del r
            torch.cuda.empty_cache()
    t0 = time.perf_counter()  # the clock sampler sees the largest batch under load
    while time.perf_counter() - t0 < 1.0:
        for _ in range(20):
            last.step()
        torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    del last
    torch.cuda.empty_cache()
    return {"workload": "Llama-2-7B-shaped MHA decode, 32/32 heads, d 128, len U[128,2048], "
                        "fused write + decode step", "unit": UNIT, "rows": rows,
            "clocks": clocks}


def run_gpu(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    from paged_kv_cache_459_b200 import pkv

    r = Resident(args, args.config, args.seed + rank, dev, batch=args.batch, cascade=args.cascade,
                 variant=args.variant, partition=args.partition, host_copies=True)
    B, hq, hkv, d, W = r.B, r.hq, r.hkv, r.d, r.W
    K, Wm = args.steps, args.warmup
    stream = torch.cuda.current_stream(dev)
    sampler = ClockSampler(device_pci_id(dev)) if rank == 0 else None
    m = timed_decode(r, K, Wm, world=world, sampler=sampler,
                     flush=True if args.flush_l2 else None)
    total_ms = m["total_ms"]
    clocks = m["clocks"]
    fused = r.fused
    unfused = None
    if fused:  # the same step as two calls (write, then decode), for comparison
        if m["flush"]:  # timed as the fused step was: rotating over copies of the pool
            r.add_cache_copies(m["cache_copies"] - 1)
            for _ in range(2 * m["cache_copies"]):
                r.next_cache()
                r.two_calls()
            uw_ms = rotating_steps(r, K, dev, r.write)
            loop = rotating_steps(r, K, dev, r.two_calls)
            r.drop_cache_copies()
            uw, per = [uw_ms / K] * K, [loop / K] * K
        else:
            _, uw_ms = device_steps(r.write, K, dev)  # the write call alone
            uw = [uw_ms / K] * K
            per, loop = device_steps(r.two_calls, K, dev)
        u_ms = max_over_ranks([loop], device=dev)[0]
        unfused = {"step_us": 1e3 * statistics.fmean(per), "write_us": 1e3 * statistics.fmean(uw),
                   "value": job_throughput(B, K, world, u_ms),
                   "how": "write + decode calls per step; write_us from K writes alone back to back"}

    # End to end through the public API: every step's inputs (q, new K/V, tables, lengths,
    # slots) go host -> device from one pinned staging buffer, and its output comes back.
    # Two device input/output sets and a copy stream let step i+1's upload and step i's
    # download overlap step i's kernels.
    parts = [(n, r.host[n]) for n in ("q", "k", "v", "tables", "lens")]
    if not fused:  # the fused step takes each token's slot from its table
        parts.append(("slots", r.host["slots"]))
    offs, total = {}, 0
    for name, t in parts:
        offs[name] = total
        total += (t.numel() * t.element_size() + 255) // 256 * 256
    stage_h = torch.empty(total, dtype=torch.uint8).pin_memory()
    for name, t in parts:
        n = t.numel() * t.element_size()
        stage_h[offs[name]:offs[name] + n].copy_(t.reshape(-1).view(torch.uint8))
    h2d = total

    def views(buf):
        v = {}
        for name, t in parts:
            n = t.numel() * t.element_size()
            v[name] = buf[offs[name]:offs[name] + n].view(t.dtype).view(t.shape)
        return v

    stage_d = [torch.empty(total, dtype=torch.uint8, device=dev) for _ in range(2)]
    sets = [views(b) for b in stage_d]
    outs = [torch.empty_like(r.out) for _ in range(2)]
    outs_h = [torch.empty(r.out.shape, dtype=r.out.dtype).pin_memory() for _ in range(2)]
    d2h = outs_h[0].numel() * outs_h[0].element_size()
    copy_stream = torch.cuda.Stream(dev)   # uploads
    d2h_stream = torch.cuda.Stream(dev)    # downloads, on the other copy engine
    h2d_done, comp_done, d2h_done = ([torch.cuda.Event(), torch.cuda.Event()] for _ in range(3))

    # the fused step through the binding's prepared form (checks done once per
    # buffer set), as a serving loop that reuses its buffers calls it
    prepared = None
    if fused and not args.cascade:
        prepared = [pkv.prepare_decode_step(outs[k], sets[k]["q"], sets[k]["k"], sets[k]["v"], r.kc,
                                            r.vc, sets[k]["tables"], sets[k]["lens"], r.scale, hkv,
                                            variant=r.variant, partition_tokens=r.partition,
                                            workspace=r.ws, err=r.err) for k in range(2)]

    def step_on(i):
        if prepared is not None:
            prepared[i % 2]()
        else:
            r.step(sets[i % 2], outs[i % 2])

    def pipelined(run_step, n=K) -> float:
        """n steps: upload of step i+1 and download of step i (two copy streams,
        one per direction) overlap step i's kernels; returns the device time of
        the whole loop (ms)."""
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        e2e_ev = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
        e2e_ev[0].record(stream)
        copy_stream.wait_stream(stream)
        with torch.cuda.stream(copy_stream):
            stage_d[0].copy_(stage_h, non_blocking=True)
            h2d_done[0].record(copy_stream)
        for i in range(n):
            cur, nxt = i % 2, (i + 1) % 2
            stream.wait_event(h2d_done[cur])
            if i >= 2:
                stream.wait_event(d2h_done[cur])  # the output buffer's previous read is done
            run_step(i)
            comp_done[cur].record(stream)
            if i + 1 < n:
                with torch.cuda.stream(copy_stream):
                    if i >= 1:
                        copy_stream.wait_event(comp_done[nxt])  # its inputs were consumed
                    stage_d[nxt].copy_(stage_h, non_blocking=True)
                    h2d_done[nxt].record(copy_stream)
            with torch.cuda.stream(d2h_stream):
                d2h_stream.wait_event(comp_done[cur])
                outs_h[cur].copy_(outs[cur], non_blocking=True)
                d2h_done[cur].record(d2h_stream)
        stream.wait_stream(copy_stream)
        stream.wait_stream(d2h_stream)
        e2e_ev[1].record(stream)
        torch.cuda.synchronize(dev)
        r.check_err("after the end-to-end steps")
        # the end-to-end steps ran the same inputs through staged copies: the
        # kernels are deterministic, so the output read back must match bit for bit
        if n > 0 and not torch.equal(outs_h[(n - 1) % 2].view(torch.int16),
                                     r.out.cpu().view(torch.int16)):
            raise SystemExit("end-to-end output differs from the device-timed output")
        return e2e_ev[0].elapsed_time(e2e_ev[1])

    # an untimed pass of the same loop first (its first steps pay for the first use of
    # the copy streams, events and staging buffers), then the K timed steps
    pipelined(step_on, max(3, Wm))
    e2e_ms = pipelined(step_on)
    # The same loop with each step's write + decode replayed from a CUDA graph
    # (one per input/output buffer set), as serving engines run decode: the
    # host no longer issues the launches one by one.
    graphs = []
    for bset in range(2):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step_on(bset)
        graphs.append(g)
    pipelined(lambda i: graphs[i % 2].replay(), max(3, Wm))
    e2e_graph_ms = pipelined(lambda i: graphs[i % 2].replay())
    del graphs
    e2e_ms, e2e_graph_ms = max_over_ranks([e2e_ms, e2e_graph_ms], device=dev)

    ab = m["bytes"]
    line = {
        "metric": METRIC, "value": m["value"], "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": Wm, "ms_per_step": total_ms / K, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {
            "workload": WORKLOAD_NAMES[args.config], "name": args.config, "batch": B,
            "num_heads": hq, "num_kv_heads": hkv, "head_dim": d, "block_tokens": 16,
            "tokens": ab["tokens"], "num_blocks": r.w.num_blocks, "table_width": W,
            "variant": r.variant_text(),
            "logical_kv_bytes": ab["kv"],
            "l2": (f"inputs smaller than L2 (KV {ab['kv'] / 1e9:.3f} GB per step): each step runs "
                   f"on the next of {m['cache_copies']} copies of the K/V pool (over 3 L2 sizes, "
                   f"as a model's layers each read their own cache), K steps back to back; the "
                   f"'flushed' key times each step alone after an L2 flush") if m["flush"] else
                  f"inputs larger than L2 (KV {ab['kv'] / 1e9:.2f} GB per step vs 126 MB L2), no flush",
            "timing": "K steps back to back between two CUDA events on the launching stream; a "
                      "spin kernel before the first lets the host enqueue ahead of the device",
            "parallelism": f"{world} independent replicas (batch per GPU fixed)",
            "seed": args.seed,
        },
        "kv_hbm_gbs": m["kv_hbm_gbs"],
        "kv_frac_of_8tbs": m["kv_frac_of_8tbs"],
        "kv_frac_of_measured_copy": m["kv_frac_of_measured_copy"],
        "write_us": None if fused else unfused and unfused["write_us"],
        "decode_us": m["step_us"],
        "step": ("pkv_paged_decode_prefix_step" if args.cascade else "pkv_paged_decode_step") +
                ": the write fused into the decode kernel" if fused else
                "pkv_paged_kv_write, then the decode call",
        "unfused": unfused,
        "flushed": flushed_key(m) if m["flush"] else None,
        "roofline": m["roofline"],
        "gpu_launches": K * r.launches_per_step(),
        "e2e": {"value": job_throughput(B, K, world, e2e_ms), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms / K,
                "how": "one pinned staging buffer per step in, output out; double-buffered, "
                       "uploads and downloads on their own streams, overlapping the kernels; K "
                       "steps timed after an untimed pass of max(3, W) steps of the same loop" +
                       ("; the step through pkv.prepare_decode_step (argument checks once per "
                        "buffer set)" if prepared is not None else "")},
        "e2e_graph": {"value": job_throughput(B, K, world, e2e_graph_ms), "unit": UNIT,
                      "ms_per_step": e2e_graph_ms / K,
                      "how": "the same loop, each step replayed from a CUDA graph"},
        "clocks": clocks,
    }
    w_host = r.w
    del r, stage_d, sets, outs
    torch.cuda.empty_cache()
    if rank == 0 and world == 1 and not args.no_extras and args.batch is None \
            and not args.cascade and args.variant == "auto":
        extra = {}
        for name in ("llama", "long"):
            if name != args.config:
                extra[name] = workload_key(args, name, dev=dev)
        extra["prefix_cascade"] = workload_key(args, "prefix", dev=dev, cascade=True)
        line["workloads"] = extra
        line["batch_sweep"] = batch_sweep_key(args, dev)
        line["prefill"] = {c: prefill_numbers(args, c, dev) for c in ("llama", "qwen")}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w_host, args.cpu_seconds)
    del w_host
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def prefill_numbers(args, config: str, dev) -> dict:
    """Paged prefill attention (tcgen05) on 4 prompts x 2048 tokens with
    Llama-2-7B-shaped (32/32) or Qwen2.5-7B-shaped (28/4) heads: TFLOP/s of the
    causal attention against the measured bf16 matmul peak, and the prompt's
    K/V write."""
    import torch

    from paged_kv_cache_459_b200 import pkv
    import workloads as wl

    steps, warm = args.steps, max(3, args.warmup)
    up = lambda b: torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).view(torch.bfloat16).to(dev)  # noqa: E731
    cfg = wl.config(config)
    hq, hkv, d, B, n = cfg["num_heads"], cfg["num_kv_heads"], cfg["head_dim"], 4, 2048
    alloc = pkv.BlockAllocator(B * n // 16 + 8, wl.rng(args.seed).permutation(B * n // 16 + 8))
    slots = []
    for b in range(B):
        alloc.add_seq(b, 0)
        slots.append(alloc.extend(b, n))
    tables, lens = alloc.export(list(range(B)), n // 16)
    nb = alloc.num_blocks
    kc, vc = up(wl.bf16_normal((nb, hkv, 16, d), args.seed, 1)), up(wl.bf16_normal((nb, hkv, 16, d), args.seed, 2))
    T = B * n
    q = up(wl.bf16_normal((T, hq, d), args.seed, 3))
    k_new, v_new = up(wl.bf16_normal((T, hkv, d), args.seed, 4)), up(wl.bf16_normal((T, hkv, d), args.seed, 5))
    out = torch.empty_like(q)
    t_d, l_d = torch.from_numpy(tables).to(dev), torch.from_numpy(lens).to(dev)
    qs = torch.tensor([b * n for b in range(B + 1)], dtype=torch.int32, device=dev)
    sl = torch.from_numpy(np.concatenate(slots)).to(dev)
    wr_ms = _events_time(lambda: pkv.paged_kv_write(k_new, v_new, kc, vc, sl), steps, warm)
    run = lambda: pkv.paged_attention_prefill(out, q, kc, vc, t_d, l_d, qs, cfg["scale"], hkv, n)  # noqa: E731
    sampler = ClockSampler(device_pci_id(dev))
    ms = _events_time(run, steps, warm)
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < 1.0:
        for _ in range(20):
            run()
        torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    flops = B * 4.0 * d * hq * n * (n + 1) / 2  # causal: row i sees i + 1 keys
    peak, kind = measured_peak_tensor()
    ach = flops / (ms * 1e-3) / 1e12
    return {"metric": "paged prefill attention TFLOP/s (causal, bf16 in / fp32 accumulate)",
            "value": ach, "unit": "TFLOP/s", "ms_per_step": ms, "steps": steps,
            "workload": f"{B} prompts x {n} tokens, {hq}/{hkv} heads, d {d}",
            "prompt_write_gbs": T * hkv * d * 2 * 2 * 2 / (wr_ms * 1e-3) / 1e9,
            "roofline": {"bound": "tensor", "achieved": ach, "peak": peak, "unit": "TFLOP/s",
                         "frac": ach / peak, "peak_kind": kind,
                         "frac_of_sustained": ach / measured_peak_tensor_sustained(),
                         "kernel": "paged_prefill_tc_kernel (tcgen05, TMEM accumulators)",
                         "traffic": committed_traffic("paged_prefill_tc_kernel",
                                                      f"prefill_{config}_4x2048"),
                         "algorithmic_flops_per_launch": flops},
            "clocks": clocks, "gpu_launches": steps}


def measured_peak_tensor_sustained() -> float:
    """The seconds-long cuBLAS figure (power-capped clocks), for context."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops_sustained"])
    except (OSError, KeyError, ValueError):
        return 1400.0


def measured_peak_tensor():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except (OSError, KeyError, ValueError):
        return 1590.0, "fallback"


def _events_time(fn, steps, warmup):
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(steps):
        fn()
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / steps  # ms


def run_alloc_row(args):
    """Host cost of the block allocator per decode step (one new token for
    every sequence of the workload, then the tables and lengths exported), on
    the CPU: what the engine pays before each decode call."""
    from paged_kv_cache_459_b200 import pkv
    import workloads as wl

    cfg = wl.config("qwen" if args.config == "qwen" else "llama")
    B = cfg["batch"]
    rng = wl.rng(args.seed)
    lens = rng.integers(cfg["len_lo"], cfg["len_hi"] + 1, size=B)
    steps, warm = args.steps, max(3, args.warmup)
    need = int(sum(-(-(int(n) + steps + warm) // 16) for n in lens))
    alloc = pkv.BlockAllocator(need + 64, rng.permutation(need + 64))
    for b, n in enumerate(lens):
        alloc.add_seq(b, int(n))
    ids = list(range(B))
    width = -(-int(lens.max() + steps + warm) // 16)
    for _ in range(warm):
        alloc.append_tokens(ids)
        alloc.export(ids, width)
    t0 = time.perf_counter()
    for _ in range(steps):
        alloc.append_tokens(ids)
        alloc.export(ids, width)
    el = time.perf_counter() - t0
    # the same steps for an engine that keeps its host tables: append_tokens_into
    # patches the entries a step changes in the exported tables
    alloc2 = pkv.BlockAllocator(need + 64, wl.rng(args.seed + 1).permutation(need + 64))
    for b, n in enumerate(lens):
        alloc2.add_seq(b, int(n))
    ids_np = np.arange(B, dtype=np.int64)
    tables, lens_h = alloc2.export(ids_np, width)
    for _ in range(warm):
        alloc2.append_tokens_into(ids_np, tables, lens_h)
    t0 = time.perf_counter()
    for _ in range(steps):
        alloc2.append_tokens_into(ids_np, tables, lens_h)
    el_into = time.perf_counter() - t0
    print(json.dumps({"row": "alloc", "steps": steps, "warmup": warm, "data": "synthetic",
                      "metric": "host allocator time per decode step (append one token to every "
                                "sequence, export tables and lengths)",
                      "value": 1e6 * el / steps, "unit": "us", "higher_is_better": False,
                      "append_into_us": 1e6 * el_into / steps,
                      "append_into": "pkv_alloc_append_tokens_into on kept host tables (only the "
                                     "changed entries written)",
                      "config": {"workload": f"{B} sequences, lengths U[{cfg['len_lo']},"
                                             f"{cfg['len_hi']}], table width {width}",
                                 "threads": 1}}), flush=True)
    return 0


def run_row(args):
    """Measurements of the rows next to the decode step: prefill attention,
    copy-on-write block copies, and block swap over the host link."""
    if args.row == "alloc":
        return run_alloc_row(args)
    import torch
    from paged_kv_cache_459_b200 import pkv
    import workloads as wl

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    steps, warm = args.steps, max(3, args.warmup)
    up = lambda b: torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).view(torch.bfloat16).to(dev)  # noqa: E731
    line = {"row": args.row, "n_gpus": 1, "steps": steps, "warmup": warm, "data": "synthetic"}
    if args.row == "prefill":
        # Qwen2.5-7B-shaped heads (default) or Llama-2-7B-shaped with --config llama, 4 x 2048
        line.update(prefill_numbers(args, "llama" if args.config == "llama" else "qwen", dev))
        line["higher_is_better"] = True
    elif args.row == "cow":
        cfg = wl.config("llama")
        hkv, d, nb, n = cfg["num_kv_heads"], cfg["head_dim"], 8192, 2048
        kc = up(wl.bf16_normal((nb, hkv, 16, d), args.seed, 1))
        vc = up(wl.bf16_normal((nb, hkv, 16, d), args.seed, 2))
        perm = wl.rng(args.seed).permutation(nb)
        src = torch.from_numpy(perm[:n].copy()).to(dev)
        dst = torch.from_numpy(perm[n:2 * n].copy()).to(dev)
        ms = _events_time(lambda: pkv.copy_blocks(kc, vc, src, dst), steps, warm)
        nbytes = n * hkv * 16 * d * 2 * 2 * 2  # read + write, K and V
        peak, kind = measured_peak_hbm()
        ach = nbytes / (ms * 1e-3) / 1e9
        line.update(metric="copy-on-write block copy GB/s (read + write)", value=ach, unit="GB/s",
                    ms_per_step=ms, higher_is_better=True,
                    config={"workload": f"{n} random block pairs, {hkv} KV heads x 16 x {d} bf16"},
                    roofline={"bound": "hbm", "achieved": ach, "peak": peak, "unit": "GB/s",
                              "frac": ach / peak, "peak_kind": kind})
    else:  # swap
        cfg = wl.config("llama")
        hkv, d, nb, n = cfg["num_kv_heads"], cfg["head_dim"], 4096, 1024
        kc = up(wl.bf16_normal((nb, hkv, 16, d), args.seed, 1))
        vc = up(wl.bf16_normal((nb, hkv, 16, d), args.seed, 2))
        hk = torch.empty((n, hkv, 16, d), dtype=torch.bfloat16).pin_memory()
        hv = torch.empty_like(hk).pin_memory()
        g = torch.from_numpy(wl.rng(args.seed).permutation(nb)[:n].copy()).to(dev)
        h = torch.arange(n, dtype=torch.int64, device=dev)
        ms_out = _events_time(lambda: pkv.swap_blocks(kc, vc, hk, hv, g, h, pkv.SWAP_OUT), steps, warm)
        ms_in = _events_time(lambda: pkv.swap_blocks(kc, vc, hk, hv, g, h, pkv.SWAP_IN), steps, warm)
        nbytes = n * hkv * 16 * d * 2 * 2
        line.update(metric="block swap GB/s over the host link (out, in)",
                    value=nbytes / (ms_out * 1e-3) / 1e9, unit="GB/s", ms_per_step=ms_out,
                    higher_is_better=True, swap_in_gbs=nbytes / (ms_in * 1e-3) / 1e9,
                    config={"workload": f"{n} blocks of {hkv} KV heads x 16 x {d} bf16, K and V "
                                        f"({nbytes / 1e6:.0f} MB each way), pinned host memory"})
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    if args.row != "decode":
        return run_row(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
