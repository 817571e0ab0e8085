#!/usr/bin/env python
"""Benchmark of the paged KV-cache decode step on B200.

One step = the whole hot path over one batch: the cache write of every
sequence's new token (pkv_paged_kv_write) and single-query decode attention
over the paged cache (pkv_paged_attention_decode).  Block tables and slots
come from the library's C++ block allocator; values are seeded synthetic bf16
N(0,1) draws.  Prints ONE JSON line (rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config llama]
    python bench.py --impl reference ...     # the fp64 CPU oracle, timed on host cores

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
    ap.add_argument("--config", choices=sorted(WORKLOAD_NAMES), default="llama")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--batch", type=int, default=None,
                    help="override the workload's batch (smaller cases for ncu captures)")
    ap.add_argument("--variant", choices=["auto", "single", "split", "stream"], default="auto")
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
    import workloads as wl

    w = wl.build(args.config, args.seed + rank, pkv.BlockAllocator, batch=args.batch)
    cfg = w.cfg
    B, hq, hkv, d = cfg["batch"], cfg["num_heads"], cfg["num_kv_heads"], cfg["head_dim"]

    def up(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)

    q_h, k_h, v_h = (up(x).pin_memory() for x in (w.q, w.k_new, w.v_new))
    tables_h = torch.from_numpy(w.block_tables).pin_memory()
    lens_h = torch.from_numpy(w.lens.astype(np.int32)).pin_memory()
    slots_h = torch.from_numpy(w.slot_mapping).pin_memory()
    kc = up(w.k_cache).to(dev)
    vc = up(w.v_cache).to(dev)
    q, k_new, v_new = q_h.to(dev), k_h.to(dev), v_h.to(dev)
    tables, lens, slots = tables_h.to(dev), lens_h.to(dev), slots_h.to(dev)
    out = torch.empty_like(q)
    out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    variant = {"auto": pkv.DECODE_AUTO, "single": pkv.DECODE_SINGLE, "split": pkv.DECODE_SPLIT,
               "stream": pkv.DECODE_STREAM}[args.variant]
    W = w.block_tables.shape[1]
    ws_bytes = pkv.decode_workspace_bytes_for(variant, B, hq, hkv, d, W, args.partition)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
    chosen = variant if variant != pkv.DECODE_AUTO else pkv.decode_variant_for(
        B, hq, hkv, d, W, args.partition, ws.numel())
    if args.cascade:
        pb_h, offs_h, mem_h = w.alloc.prefix_groups(list(range(B)))
        pb, offs_g, mem = (torch.from_numpy(x).to(dev) for x in (pb_h, offs_h, mem_h))
        suffix_bound = pkv.suffix_blocks_bound(w.lens, pb_h)  # the allocator's host view
        ws = torch.empty(pkv.decode_prefix_workspace_bytes(B, hq, d, W, args.partition),
                         dtype=torch.uint8, device=dev)
    scale = cfg["scale"]

    def write():
        pkv.paged_kv_write(k_new, v_new, kc, vc, slots, err=err)

    def decode():
        if args.cascade:
            pkv.paged_attention_decode_prefix(out, q, kc, vc, tables, lens, scale, hkv, pb, offs_g, mem,
                                              max_suffix_blocks=suffix_bound,
                                              partition_tokens=args.partition, workspace=ws,
                                              err=err)
        else:
            pkv.paged_attention_decode(out, q, kc, vc, tables, lens, scale, hkv, variant=variant,
                                       partition_tokens=args.partition, workspace=ws, err=err)

    # The step: the new token's K/V write fused into the decode kernel
    # (pkv_paged_decode_step), or the write and the decode as two calls.
    fused = not args.unfused and (args.cascade or chosen != pkv.DECODE_STREAM)

    def fused_step(o=None, c=None):
        c = c or {"q": q, "k": k_new, "v": v_new, "tables": tables, "lens": lens}
        if args.cascade:
            pkv.paged_decode_prefix_step(out if o is None else o, c["q"], c["k"], c["v"], kc, vc,
                                         c["tables"], c["lens"], scale, hkv, pb, offs_g, mem,
                                         max_suffix_blocks=suffix_bound,
                                         partition_tokens=args.partition, workspace=ws, err=err)
        else:
            pkv.paged_decode_step(out if o is None else o, c["q"], c["k"], c["v"], kc, vc,
                                  c["tables"], c["lens"], scale, hkv, variant=variant,
                                  partition_tokens=args.partition, workspace=ws, err=err)

    def step():
        if fused:
            fused_step()
        else:
            write()
            decode()

    stream = torch.cuda.current_stream(dev)
    K, Wm = args.steps, args.warmup
    for _ in range(Wm):
        step()
        if fused:
            write()
            decode()
    torch.cuda.synchronize(dev)
    if int(err.item()) != 0:
        raise SystemExit(f"device error word {int(err.item())} after warm-up")

    sampler = ClockSampler(device_pci_id(dev)) if rank == 0 else None
    flush = args.flush_l2 or algorithmic_bytes(w)["kv"] <= L2_BYTES
    flush_buf = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev) if flush else None
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    t_start.record(stream)
    for i in range(K):
        if flush:
            flush_buf.zero_()  # L2 holds none of this step's inputs
        ev[i][0].record(stream)
        if fused:
            fused_step()
        else:
            write()
            ev[i][1].record(stream)
            decode()
        ev[i][2].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    total_ms = t_start.elapsed_time(t_end)
    if flush:  # the flushes are not the step's work: sum the steps' own events
        total_ms = sum(e[0].elapsed_time(e[2]) for e in ev)
    if fused:  # one call: the decode kernel's time includes the write
        write_ms = None
        decode_ms = statistics.fmean(e[0].elapsed_time(e[2]) for e in ev)
    else:
        write_ms = statistics.fmean(e[0].elapsed_time(e[1]) for e in ev)
        decode_ms = statistics.fmean(e[1].elapsed_time(e[2]) for e in ev)
    unfused = None
    if fused:  # the same step as two calls, for comparison
        uev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
        torch.cuda.synchronize(dev)
        for i in range(K):
            if flush:
                flush_buf.zero_()
            uev[i][0].record(stream)
            write()
            uev[i][1].record(stream)
            decode()
            uev[i][2].record(stream)
        torch.cuda.synchronize(dev)
        unfused = {"write_us": 1e3 * statistics.fmean(e[0].elapsed_time(e[1]) for e in uev),
                   "decode_us": 1e3 * statistics.fmean(e[1].elapsed_time(e[2]) for e in uev),
                   "total_ms": sum(e[0].elapsed_time(e[2]) for e in uev)}
    prefix_tc = None
    if args.cascade and fused:  # the prefix chunks on mma.sync (default) and on tcgen05, one loop each
        prefix_tc = {"default_step_us": 1e3 * _events_time(step, K, Wm)}
        os.environ["PKV_CASCADE_TC"] = "1"
        try:
            prefix_tc["step_us"] = 1e3 * _events_time(step, K, Wm)
        finally:
            os.environ.pop("PKV_CASCADE_TC")
        prefix_tc["how"] = ("K steps back to back between two events, mma.sync prefix chunks "
                            "(default_step_us) then PKV_CASCADE_TC=1 (step_us)")
    # keep the GPU loaded long enough for the clock sampler to see it
    if sampler is not None:
        t0 = time.perf_counter()
        while time.perf_counter() - t0 < 1.0:
            for _ in range(50):
                step()
            torch.cuda.synchronize(dev)
    clocks = sampler.stop() if sampler is not None else None

    # End to end through the public API: every step's inputs (q, new K/V, tables, lengths,
    # slots) go host -> device from one pinned staging buffer, and its output comes back.
    # Two device input/output sets and a copy stream let step i+1's upload and step i's
    # download overlap step i's kernels.
    parts = [("q", q_h), ("k", k_h), ("v", v_h), ("tables", tables_h), ("lens", lens_h)]
    if not fused:  # the fused step takes each token's slot from its table
        parts.append(("slots", slots_h))
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
    outs = [torch.empty_like(out) for _ in range(2)]
    outs_h = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    d2h = outs_h[0].numel() * outs_h[0].element_size()
    copy_stream = torch.cuda.Stream(dev)   # uploads
    d2h_stream = torch.cuda.Stream(dev)    # downloads, on the other copy engine
    h2d_done, comp_done, d2h_done = ([torch.cuda.Event(), torch.cuda.Event()] for _ in range(3))

    def step_on(i):
        c = sets[i % 2]
        o = outs[i % 2]
        if fused:
            fused_step(o, c)
            return
        pkv.paged_kv_write(c["k"], c["v"], kc, vc, c["slots"], err=err)
        if args.cascade:
            pkv.paged_attention_decode_prefix(o, c["q"], kc, vc, c["tables"], c["lens"], scale, hkv,
                                              pb, offs_g, mem, max_suffix_blocks=suffix_bound,
                                              partition_tokens=args.partition, workspace=ws,
                                              err=err)
        else:
            pkv.paged_attention_decode(o, c["q"], kc, vc, c["tables"], c["lens"], scale, hkv,
                                       variant=variant, partition_tokens=args.partition,
                                       workspace=ws, err=err)

    def pipelined(run_step) -> float:
        """K steps: upload of step i+1 and download of step i (two copy streams,
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
        for i in range(K):
            cur, nxt = i % 2, (i + 1) % 2
            stream.wait_event(h2d_done[cur])
            if i >= 2:
                stream.wait_event(d2h_done[cur])  # the output buffer's previous read is done
            run_step(i)
            comp_done[cur].record(stream)
            if i + 1 < K:
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
        if int(err.item()) != 0:
            raise SystemExit(f"device error word {int(err.item())} after the timed steps")
        # the end-to-end steps ran the same inputs through staged copies: the
        # kernels are deterministic, so the output read back must match bit for bit
        if K > 0 and not torch.equal(outs_h[(K - 1) % 2].view(torch.int16),
                                     out.cpu().view(torch.int16)):
            raise SystemExit("end-to-end output differs from the device-timed output")
        return e2e_ev[0].elapsed_time(e2e_ev[1])

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
    e2e_graph_ms = pipelined(lambda i: graphs[i % 2].replay())
    del graphs

    total_ms, e2e_ms, e2e_graph_ms, u_ms = max_over_ranks(
        [total_ms, e2e_ms, e2e_graph_ms, unfused["total_ms"] if unfused else 0.0], device=dev)
    if unfused:
        unfused = {"write_us": unfused["write_us"], "decode_us": unfused["decode_us"],
                   "value": job_throughput(B, K, world, u_ms)}

    ab = algorithmic_bytes(w)
    peak, peak_kind = measured_peak_hbm()
    dec_bytes = ab["kv"] + ab["q"]
    if args.cascade:
        # what the cascade must read: each group's prefix once, every suffix once
        unique_tokens = int((np.asarray(w.lens, np.int64) - 16 * pb_h.astype(np.int64)).sum())
        unique_tokens += sum(16 * int(pb_h[mem_h[offs_h[g]]]) for g in range(len(offs_h) - 1))
        dec_bytes = unique_tokens * hkv * d * 2 * 2 + ab["q"]
    if fused:  # the new tokens' K/V: read once, written once
        dec_bytes += 2 * B * hkv * d * 2 * 2
    achieved = dec_bytes / (decode_ms * 1e-3) / 1e9
    value = job_throughput(B, K, world, total_ms)
    e2e_value = job_throughput(B, K, world, e2e_ms)
    # write + decode, + the merge (split-K, balanced) or the longest-first order (single pass)
    ordered = chosen == pkv.DECODE_SINGLE and ws.numel() >= 4 * B
    launches_per_step = (1 if fused else 2) + \
        (1 if chosen in (pkv.DECODE_SPLIT, pkv.DECODE_STREAM) or ordered else 0)
    if args.cascade:  # (write;) prefix chunks + suffix split-K in one launch, merge
        launches_per_step = 2 if fused else 3
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": Wm, "ms_per_step": total_ms / K, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {
            "workload": WORKLOAD_NAMES[args.config], "name": args.config, "batch": B,
            "num_heads": hq, "num_kv_heads": hkv, "head_dim": d, "block_tokens": 16,
            "tokens": ab["tokens"], "num_blocks": w.num_blocks, "table_width": W,
            "variant": {pkv.DECODE_SINGLE: "single pass (one CTA per sequence x KV head, longest "
                                            "first)" if ordered else
                        "single pass (one CTA per sequence x KV head)",
                        pkv.DECODE_SPLIT: "split-K %d-token partitions + merge" % args.partition,
                        pkv.DECODE_STREAM: "balanced stream-K (equal tile ranges per warp) + merge",
                        }[chosen] if not args.cascade else
            "shared-prefix cascade (prefix once per group x KV head, split-K suffixes, merge)",
            "logical_kv_bytes": ab["kv"],
            "l2": (f"L2 flushed between steps (256 MB write); step time from per-step events "
                   f"(KV {ab['kv'] / 1e9:.3f} GB per step)") if flush else
                  f"inputs larger than L2 (KV {ab['kv'] / 1e9:.2f} GB per step vs 126 MB L2), no flush",
            "parallelism": f"{world} independent replicas (batch per GPU fixed)",
            "seed": args.seed,
        },
        "kv_hbm_gbs": achieved,
        "kv_frac_of_8tbs": achieved / NOMINAL_HBM_GBS,
        "kv_frac_of_measured_copy": achieved / peak,
        "write_us": write_ms * 1e3 if write_ms is not None else None,
        "decode_us": decode_ms * 1e3,
        "step": ("pkv_paged_decode_prefix_step" if args.cascade else "pkv_paged_decode_step") +
                ": the write fused into the decode kernel" if fused else
                "pkv_paged_kv_write, then the decode call",
        "unfused": unfused,
        **({"prefix_tcgen05": prefix_tc} if prefix_tc else {}),
        "roofline": {
            "bound": "hbm",
            "kernel": ("cascade_kernel (prefix chunks + suffix units" +
                       (", fused write" if fused else "") + ") + cascade_merge_kernel")
                      if args.cascade else
                      ("paged_decode_kernel with the fused write" if fused else "paged_decode_kernel")
                      + (" + merge kernel" if chosen == pkv.DECODE_SPLIT else
                         " + order kernel" if ordered else ""),
            "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
            "peak_kind": peak_kind,
            "traffic": committed_traffic("paged_decode_kernel", args.config),
            "algorithmic_bytes_per_launch": dec_bytes,
        },
        "gpu_launches": K * launches_per_step,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms / K,
                "how": "one pinned staging buffer per step in, output out; double-buffered, "
                       "uploads and downloads on their own streams, overlapping the kernels"},
        "e2e_graph": {"value": job_throughput(B, K, world, e2e_graph_ms), "unit": UNIT,
                      "ms_per_step": e2e_graph_ms / K,
                      "how": "the same loop, each step replayed from a CUDA graph"},
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


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
        # Llama-2-7B-shaped heads (or Qwen2.5-7B-shaped with --config qwen), 4 prompts x 2048
        cfg = wl.config("qwen" if args.config == "qwen" else "llama")
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
        os.environ["PKV_PREFILL_WARP_MMA"] = "1"
        ms_warp = _events_time(run, steps, warm)
        os.environ.pop("PKV_PREFILL_WARP_MMA")
        ms = _events_time(run, steps, warm)
        flops = B * 4.0 * d * hq * n * (n + 1) / 2  # causal: row i sees i + 1 keys
        peak, kind = measured_peak_tensor()
        ach = flops / (ms * 1e-3) / 1e12
        line.update(metric="paged prefill attention TFLOP/s (causal, bf16 in / fp32 accumulate)",
                    value=ach, unit="TFLOP/s", ms_per_step=ms, higher_is_better=True,
                    config={"workload": f"{B} prompts x {n} tokens, {hq}/{hkv} heads, d {d}"},
                    prompt_write_gbs=T * hkv * d * 2 * 2 * 2 / (wr_ms * 1e-3) / 1e9,
                    warp_mma_tflops=flops / (ms_warp * 1e-3) / 1e12,
                    roofline={"bound": "tensor", "achieved": ach, "peak": peak, "unit": "TFLOP/s",
                              "frac": ach / peak, "peak_kind": kind,
                              "frac_of_sustained": ach / measured_peak_tensor_sustained(),
                              "kernel": "paged_prefill_tc_kernel (tcgen05, TMEM accumulators)",
                              "traffic": committed_traffic(
                                  "paged_prefill_tc_kernel",
                                  "prefill_qwen_4x2048" if args.config == "qwen" else "prefill_llama_4x2048")})
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
