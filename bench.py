#!/usr/bin/env python
"""Throughput of the fused 2D Neighborhood Attention forward (na2d_forward).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload stage1] [--impl ours|reference]

One step is one na2d_forward call over one batch of the workload (default:
NAT-Tiny level-1 map, B=32 heads=2 H=W=56 d=32 k=7 bf16).  With N > 1 the
script is launched once per GPU by torch.distributed.run; every rank runs
the same per-GPU batch on its own GPU (weak scaling, no collective on the
data path) and `value` counts the query-neighbours of all ranks over the
slowest rank's time.

Timed region: W untimed warm-up steps, then exactly K steps replayed from
CUDA graphs, bracketed by a barrier and a device synchronize, timed with
CUDA events on the launching stream.  Steps cycle through R input/output
sets whose total size is at least 3x the L2 cache, so every step reads its
inputs from HBM.  The line also reports an end-to-end figure through
na2d_forward_host (pinned host buffers, copies inside the timed region),
the roofline of the kernel against the measured HBM bandwidth, the SM
clocks sampled during the timed region and the fp64 CPU oracle's
throughput on the host cores (rank 0, N = 1 only).

--impl reference times the fp64 CPU oracle on the host cores instead (rank 0
only; other ranks exit at once): each step is a bounded sample of the same
workload.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "2D NA fwd query-neighbours/s (G) and % of HBM/tensor roofline on 1 B200"
UNIT = "G query-neighbours/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
TC_SOURCE = os.path.join(ROOT, "vision_sliding_window_b200", "csrc", "na2d_tc.cu")
SIMT_SOURCE = os.path.join(ROOT, "vision_sliding_window_b200", "csrc", "na2d_simt.cu")


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=100)
    ap.add_argument("--workload", default="stage1")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--graph-steps", type=int, default=250, help="steps per captured CUDA graph")
    ap.add_argument("--api", choices=["fused", "unfused"], default="fused",
                    help="unfused: time na2d_qk_rpb, na2d_softmax and na2d_av one by one instead")
    return ap.parse_args(argv)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in FALLBACK_PEAKS}, "measured"
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def file_sha(path):
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def strip_c_comments(text):
    """C/C++ source without comments and without blank or repeated whitespace:
    what the compiler sees, so an edit of comments alone keeps its hash."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c in "\"'":
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        else:
            out.append(c)
            i += 1
    lines = ("".join(out)).splitlines()
    return "\n".join(" ".join(ln.split()) for ln in lines if ln.strip())


def code_sha(path):
    """Hash of a kernel source with its comments stripped (see strip_c_comments)."""
    with open(path) as f:
        return hashlib.sha256(strip_c_comments(f.read()).encode()).hexdigest()[:16]


def profiled_traffic(kernel_source, workload):
    """DRAM bytes per launch from the committed ncu summary of this kernel and
    workload, if it was captured on code identical (comments aside) to the
    current source; else None.  A summary records the hash of the file it
    was captured on (source_sha256_16) and of its comment-free code
    (code_sha256_16); only the latter is compared."""
    name = os.path.splitext(os.path.basename(kernel_source))[0]
    path = os.path.join(ROOT, "profiles", f"{name}_{workload}.md")
    try:
        text = open(path).read()
    except OSError:
        return None
    sha = re.search(r"code_sha256_16:\s*([0-9a-f]+)", text)
    tr = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", text)
    if not sha or not tr or sha.group(1) != code_sha(kernel_source):
        return None
    return float(tr.group(1))


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi samples (every 200 ms) of the SM clock and throttle reasons."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        self.lines = []
        self.device_index = device_index
        self.window = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200",
                 "-i", str(self.device_index)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.6)

    def mark(self, t0, t1):
        self.window = (t0, t1)

    def stop(self):
        if not self.proc:
            return
        time.sleep(0.3)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self, window=None):
        """Median SM clock, max clock and active throttle reasons of the samples
        inside `window` (host time (t0, t1); default: the marked window)."""
        window = window or self.window
        rows = []
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                rows.append((ts, float(parts[2]), float(parts[3]), parts[6:10]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        inside = [r for r in rows if window and window[0] - 0.25 <= r[0] <= window[1] + 0.25]
        use, where = (inside, "timed region") if inside else (rows, "whole run (timed region shorter than a sample)")
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({n for r in use for n, a in zip(names, r[3]) if a.lower() == "active"})
        return {"sm_mhz": statistics.median(r[1] for r in use), "sm_max_mhz": max(r[2] for r in use),
                "reasons": reasons, "samples": len(use), "window": where}


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


# ------------------------------------------------------------- CPU oracle

def cpu_oracle_throughput(w, seconds):
    """Times the fp64 oracle on a bounded sample of the workload: with all
    host threads, passes over all (b, h) maps, or over as many as one pass of
    about `seconds` allows, repeated until `seconds` have passed; then with
    one thread on one map for about a tenth of that."""
    import oracle
    from vision_sliding_window_b200.inputs import workload_inputs

    q, k, v, rpb = workload_inputs(w)
    q, k, v = (t.double().numpy() for t in (q, k, v))
    rpb = rpb.double().numpy()
    nthreads = oracle.max_threads()
    maps = w.B * w.heads
    # warm the thread pool on one map, then size the sample
    oracle.forward_rows(q, k, v, rpb, w.ks, 0, w.H, nthreads)
    t0 = time.perf_counter()
    oracle.forward_rows(q, k, v, rpb, w.ks, 0, w.H, nthreads)
    per_map = max(time.perf_counter() - t0, 1e-6)
    n_maps = max(1, min(maps, int(seconds / per_map)))
    passes = 0
    t0 = time.perf_counter()
    while True:
        oracle.forward_rows(q, k, v, rpb, w.ks, 0, n_maps * w.H, nthreads)
        passes += 1
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    qn = passes * n_maps * w.H * w.W * w.ks * w.ks
    sample = (f"{passes} pass(es) over {n_maps} of {maps} (b, h) maps of {w.name} "
              f"({qn / 1e6:.2f} M query-neighbours, {dt:.1f} s)")
    # one thread: whole maps until a tenth of the budget has passed
    rows1, t1 = 0, time.perf_counter()
    while True:
        oracle.forward_rows(q, k, v, rpb, w.ks, 0, w.H, 1)
        rows1 += w.H
        if time.perf_counter() - t1 >= seconds / 10:
            break
    dt1 = time.perf_counter() - t1
    qn1 = rows1 * w.W * w.ks * w.ks
    return {"value": qn / dt / 1e9, "unit": UNIT, "cores": nthreads, "kind": "oracle", "sample": sample,
            "cpu_model": cpu_model(),
            "one_thread": {"value": qn1 / dt1 / 1e9, "unit": UNIT,
                           "sample": f"{rows1 // w.H} map(s) of {w.name}, {dt1:.1f} s"}}


def run_reference(args, rank):
    from vision_sliding_window_b200.inputs import WORKLOADS

    if rank != 0:
        return 0
    import oracle

    w = WORKLOADS[args.workload]
    from vision_sliding_window_b200.inputs import workload_inputs

    q, k, v, rpb = workload_inputs(w)
    q, k, v = (t.double().numpy() for t in (q, k, v))
    rpb = rpb.double().numpy()
    nthreads = oracle.max_threads()
    t0 = time.perf_counter()
    oracle.forward_rows(q, k, v, rpb, w.ks, 0, w.H, nthreads)
    per_map = max(time.perf_counter() - t0, 1e-6)
    budget = min(10.0, 150.0 / max(1, args.steps + args.warmup))  # seconds per step
    n_maps = max(1, min(w.B * w.heads, int(budget / per_map)))
    rows = n_maps * w.H
    for _ in range(args.warmup):
        oracle.forward_rows(q, k, v, rpb, w.ks, 0, rows, nthreads)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.forward_rows(q, k, v, rpb, w.ks, 0, rows, nthreads)
    dt = time.perf_counter() - t0
    qn_step = n_maps * w.H * w.W * w.ks * w.ks
    value = args.steps * qn_step / dt / 1e9
    sample = f"each step: {n_maps} of {w.B * w.heads} (b, h) maps of {w.name} ({qn_step / 1e6:.3f} M query-neighbours)"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(w, args.gpus),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": nthreads, "kind": "oracle", "sample": sample,
                         "cpu_model": cpu_model()},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(w, n_gpus, extra=None):
    cfg = {
        "workload": (f"{w.name}: B={w.B} heads={w.heads} H={w.H} W={w.W} d={w.d} k={w.ks} {w.dtype}, "
                     f"q/k/v ~ N(0,1){' x 1/sqrt(d)' if w.qkv_scale != 1 else ''}, rpb ~ N(0,0.02^2), seed {w.seed}"),
        "global_batch": w.B * n_gpus,
        "per_gpu_batch": w.B,
        "parallelism": f"batch-sharded x{n_gpus}, no collective" if n_gpus > 1 else "single GPU",
    }
    if extra:
        cfg.update(extra)
    return cfg


# -------------------------------------------------------------------- ours

# The headline workloads besides stage1 that the line reports, each timed in
# the same run (nested under "targets").
TARGETS = ("hires_k7", "hires_k13")
TARGET_STEPS = 400


class Timer:
    """Back-to-back na2d_forward launches of one workload, replayed from CUDA
    graphs over R rotating input/output sets (R sets >= 3x L2)."""

    def __init__(self, w, dev, rank, graph_steps):
        import torch
        from dataclasses import replace

        from vision_sliding_window_b200 import na2d
        from vision_sliding_window_b200.inputs import workload_inputs

        self.w, self.dev, self.na2d = w, dev, na2d
        # rank r holds batch entries [r*B, (r+1)*B) of the global batch (its own seed)
        self.host = workload_inputs(replace(w, seed=w.seed + rank))
        self.set_bytes = w.io_bytes
        self.l2 = torch.cuda.get_device_properties(dev).L2_cache_size
        self.R = max(2, math.ceil(3 * self.l2 / self.set_bytes))
        self.sets = []
        for _ in range(self.R):
            q, k, v, rpb = (t.to(dev) for t in self.host)
            self.sets.append((q, k, v, rpb, torch.empty_like(q)))
        self.graph_steps = graph_steps
        self.kind = na2d.forward_kernel(*w.shape(), w.ks, self.host[0].dtype)

    def step(self, i):
        q, k, v, rpb, out = self.sets[i % self.R]
        self.na2d.forward(q, k, v, rpb, self.w.ks, out=out)

    def warm(self, n):
        import torch

        for i in range(max(n, 0)):
            self.step(i)
        torch.cuda.synchronize(self.dev)
        if self.na2d.device_status() != self.na2d.NA_OK:
            raise SystemExit(f"device status not OK after warm-up of {self.w.name}")

    def timed(self, steps, barrier=None):
        """Device time (ms) of exactly `steps` launches, and the host window."""
        import torch

        G = max(1, min(self.graph_steps, steps))
        n_full, rem = divmod(steps, G)

        def capture(n):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                for i in range(n):
                    self.step(i)
            return g

        g_full = capture(G) if n_full else None
        g_rem = capture(rem) if rem else None
        if g_full is not None:
            g_full.replay()  # one untimed replay of the captured graph
        torch.cuda.synchronize(self.dev)
        stream = torch.cuda.current_stream(self.dev)
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if barrier:
            barrier(self.dev)
        torch.cuda.synchronize(self.dev)
        t0 = time.time()
        ev0.record(stream)
        for _ in range(n_full):
            g_full.replay()
        if g_rem is not None:
            g_rem.replay()
        ev1.record(stream)
        torch.cuda.synchronize(self.dev)
        t1 = time.time()
        if barrier:
            barrier(self.dev)
        status = self.na2d.device_status()
        if status != self.na2d.NA_OK:
            raise SystemExit(f"device status {self.na2d.status_str(status)} after timing {self.w.name}")
        del g_full, g_rem
        return ev0.elapsed_time(ev1), (t0, t1), G

    def release(self):
        self.sets = []


def roofline_of(w, launch_s, kernel_kind, peaks, peak_src):
    kernel_source = TC_SOURCE if kernel_kind == 1 else SIMT_SOURCE
    kernel_name = "na2d_fwd_tc" if kernel_kind == 1 else "na2d_fwd_simt"
    achieved_gbs = w.io_bytes / launch_s / 1e9
    tflops = w.flops / launch_s / 1e12
    return {
        "bound": "hbm", "achieved": achieved_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
        "frac": achieved_gbs / peaks["hbm_gbs"],
        "traffic": profiled_traffic(kernel_source, w.name),
        "traffic_kind": ("ncu dram__bytes_read.sum + dram__bytes_write.sum per launch; the output's "
                         "writes still held in L2 when the kernel ends are not counted, so this is "
                         "in effect the DRAM read traffic"),
        "kernel": kernel_name, "launch_us": launch_s * 1e6, "peak_source": peak_src,
        "algorithmic_bytes": w.io_bytes,
        "tensor_view": {"achieved_tflops": tflops, "peak_tflops": peaks["bf16_tflops"],
                        "frac": tflops / peaks["bf16_tflops"]},
    }


def run_unfused(args, w, dev, peaks, peak_src):
    """Times the unfused chain call by call: na2d_qk_rpb (q, k -> float32
    logits), na2d_softmax (in place) and na2d_av (weights, v -> out), each
    replayed from CUDA graphs over rotating input sets larger than L2, and
    reports per call the time, the algorithmic bytes it moves and the
    fraction of the HBM roofline."""
    import torch

    from vision_sliding_window_b200 import na2d
    from vision_sliding_window_b200.inputs import workload_inputs

    host = workload_inputs(w)
    es = w.elem_bytes
    tensor = w.queries * w.d * es
    attn_bytes = w.queries * w.ks * w.ks * 4
    rpb_bytes = w.heads * (2 * w.ks - 1) ** 2 * es
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    R = max(2, math.ceil(3 * l2 / (3 * tensor + attn_bytes)))
    sets = []
    for _ in range(R):
        q, k, v, rpb = (t.to(dev) for t in host)
        sets.append((q, k, v, rpb, torch.empty((*q.shape[:4], w.ks * w.ks), device=dev), torch.empty_like(q)))
    calls = {
        "na2d_qk_rpb": (lambda s: na2d.qk_rpb(s[0], s[1], s[3], w.ks, attn=s[4]), 2 * tensor + attn_bytes + rpb_bytes),
        "na2d_softmax": (lambda s: na2d.softmax_(s[4], w.ks, 1.0 / math.sqrt(w.d)), 2 * attn_bytes),
        "na2d_av": (lambda s: na2d.av(s[4], s[2], w.ks, out=s[5]), attn_bytes + 2 * tensor),
    }
    steps = max(args.steps, 20)
    res = {}
    total_us = 0.0
    for name, (fn, nbytes) in calls.items():
        for i in range(max(args.warmup, 3)):
            fn(sets[i % R])
        torch.cuda.synchronize(dev)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(steps):
                fn(sets[i % R])
        g.replay()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        g.replay()
        e1.record()
        torch.cuda.synchronize(dev)
        us = e0.elapsed_time(e1) * 1e3 / steps
        del g
        gbs = nbytes / us / 1e3
        total_us += us
        res[name] = {"us_per_call": us, "algorithmic_bytes": nbytes, "gbs": gbs, "frac": gbs / peaks["hbm_gbs"]}
    if na2d.device_status() != na2d.NA_OK:
        raise SystemExit("device status not OK after the unfused chain")
    line = {
        "metric": METRIC, "api": "unfused", "value": w.query_neighbours / (total_us * 1e-6) / 1e9, "unit": UNIT,
        "n_gpus": 1, "steps": steps, "warmup": args.warmup, "ms_per_step": total_us / 1e3,
        "higher_is_better": True, "dtype": w.dtype, "data": "synthetic",
        "config": workload_config(w, 1, {"l2": f"rotating {R} sets", "timing": "CUDA graphs, CUDA events"}),
        "calls": res, "peak_source": peak_src, "gpu_launches": 3 * steps,
    }
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    args = parse_args(argv)
    from vision_sliding_window_b200.dist import barrier, env_rank, max_over_ranks

    rank, local_rank, world = env_rank()
    if args.impl == "reference":
        return run_reference(args, rank)

    import torch
    import torch.distributed as dist

    from vision_sliding_window_b200 import na2d
    from vision_sliding_window_b200.inputs import WORKLOADS

    w = WORKLOADS[args.workload]
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    na2d.load_library()
    peaks, peak_src = load_peaks()
    if args.api == "unfused":
        if world > 1:
            raise SystemExit("--api unfused runs on one GPU")
        return run_unfused(args, w, dev, peaks, peak_src)

    sampler = ClockSampler(local_rank) if rank == 0 else None
    if sampler:
        sampler.start()

    main_timer = Timer(w, dev, rank, args.graph_steps)
    main_timer.warm(args.warmup)
    local_ms, window, G = main_timer.timed(args.steps, barrier)
    total_ms = max_over_ranks(local_ms, dev)
    if sampler:
        sampler.mark(*window)
    host = main_timer.host
    R, set_bytes, l2 = main_timer.R, main_timer.set_bytes, main_timer.l2
    kernel_kind = main_timer.kind
    main_timer.release()

    # the other headline workloads, each timed the same way (same ranks, same order)
    targets = {}
    if args.workload == "stage1":
        for name in TARGETS:
            tw = WORKLOADS[name]
            t = Timer(tw, dev, rank, args.graph_steps)
            t.warm(max(args.warmup, 3))
            n = max(args.steps, TARGET_STEPS)
            ms, win, _ = t.timed(n, barrier)
            ms = max_over_ranks(ms, dev)
            launch = ms * 1e-3 / n
            rl = roofline_of(tw, launch, t.kind, peaks, peak_src)
            targets[name] = {
                "workload": workload_config(tw, world)["workload"],
                "steps": n, "us_per_launch": launch * 1e6,
                "value": world * n * tw.query_neighbours / (ms * 1e-3) / 1e9, "unit": UNIT,
                "gbs": rl["achieved"], "frac": rl["frac"], "tflops": rl["tensor_view"]["achieved_tflops"],
                "traffic": rl["traffic"], "kernel": rl["kernel"], "window": win,
            }
            t.release()

    # end to end through the host-buffer entry point (pinned host buffers,
    # every step's copies in and out inside the timed region)
    pin = [t.pin_memory() for t in host]
    out_host = torch.empty_like(host[0]).pin_memory()
    ws = torch.empty(na2d.host_workspace_bytes(*w.shape(), w.ks, host[0].dtype), dtype=torch.uint8, device=dev)
    for _ in range(3):
        na2d.forward_host(*pin, out_host, w.ks, ws)
    torch.cuda.synchronize(dev)
    stream = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(dev)
    torch.cuda.synchronize(dev)
    e0.record(stream)
    for _ in range(args.e2e_steps):
        na2d.forward_host(*pin, out_host, w.ks, ws)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dev)
    if sampler:
        sampler.stop()

    qn_step = w.query_neighbours
    value = world * args.steps * qn_step / (total_ms * 1e-3) / 1e9
    e2e_value = world * args.e2e_steps * qn_step / (e2e_ms * 1e-3) / 1e9
    launch_s = local_ms * 1e-3 / args.steps
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": workload_config(w, world, {
            "l2": f"rotating {R} input/output sets ({R * set_bytes / 1e6:.0f} MB, L2 {l2 / 1e6:.0f} MB)",
            "timing": f"CUDA graphs of {G} steps, CUDA events on the launching stream, max over ranks",
        }),
        "roofline": roofline_of(w, launch_s, kernel_kind, peaks, peak_src),
        "e2e": {"value": e2e_value, "unit": UNIT,
                "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in host),
                "d2h_bytes_per_step": host[0].numel() * host[0].element_size(),
                "api": "na2d_forward_host", "steps": args.e2e_steps},
        "gpu_launches": args.steps,
    }
    if rank == 0:
        line["clocks"] = sampler.summary() if sampler else None
        if targets:
            for tv in targets.values():
                tv["clocks"] = sampler.summary(tv.pop("window")) if sampler else None
            line["targets"] = targets
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_oracle_throughput(w, args.cpu_seconds)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
