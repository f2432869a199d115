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


def profiled_traffic(kernel_source, workload):
    """DRAM bytes per launch from the committed ncu summary of this kernel and
    workload, if it was taken on the current source; else None."""
    name = os.path.splitext(os.path.basename(kernel_source))[0]
    path = os.path.join(ROOT, "profiles", f"{name}_{workload}.md")
    try:
        text = open(path).read()
    except OSError:
        return None
    sha = re.search(r"source_sha256_16:\s*([0-9a-f]+)", text)
    tr = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", text)
    if not sha or not tr or sha.group(1) != file_sha(kernel_source):
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

    def summary(self):
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
        inside = [r for r in rows if self.window and self.window[0] - 0.25 <= r[0] <= self.window[1] + 0.25]
        use, where = (inside, "timed region") if inside else (rows, "whole run (timed region shorter than a sample)")
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({n for r in use for n, a in zip(names, r[3]) if a.lower() == "active"})
        return {"sm_mhz": statistics.median(r[1] for r in use), "sm_max_mhz": max(r[2] for r in use),
                "reasons": reasons, "samples": len(use), "window": where}


# ------------------------------------------------------------- CPU oracle

def cpu_oracle_throughput(w, seconds, rows_per_call=None):
    """Times the fp64 oracle (all host threads) on a bounded sample of the
    workload: passes over all (b, h) maps, or over as many as one pass of
    about `seconds` allows, repeated until `seconds` have passed."""
    import oracle
    from vision_sliding_window_b200.inputs import workload_inputs

    q, k, v, rpb = workload_inputs(w)
    q, k, v = (t.double().numpy() for t in (q, k, v))
    rpb = rpb.double().numpy()
    nthreads = oracle.max_threads()
    maps = w.B * w.heads
    # warm the thread pool on one map, then size the sample: whole passes over
    # the workload (or over as many maps as fit), repeated until `seconds`
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
    return {"value": qn / dt / 1e9, "unit": UNIT, "cores": nthreads, "kind": "oracle", "sample": sample}


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
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": nthreads, "kind": "oracle", "sample": sample},
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

def main(argv=None):
    args = parse_args(argv)
    from vision_sliding_window_b200.dist import barrier, env_rank, max_over_ranks

    rank, local_rank, world = env_rank()
    if args.impl == "reference":
        return run_reference(args, rank)

    import torch
    import torch.distributed as dist

    from vision_sliding_window_b200 import na2d
    from vision_sliding_window_b200.inputs import WORKLOADS, workload_inputs

    w = WORKLOADS[args.workload]
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    lib = na2d.load_library()
    kernel_kind = na2d.forward_kernel(*w.shape(), w.ks, {"bf16": torch.bfloat16, "f16": torch.float16,
                                                         "f32": torch.float32}[w.dtype])
    kernel_source = TC_SOURCE if kernel_kind == 1 else SIMT_SOURCE
    kernel_name = "na2d_fwd_tc" if kernel_kind == 1 else "na2d_fwd_simt"

    # inputs: rank r holds batch entries [r*B, (r+1)*B) of the global batch (its own seed)
    from dataclasses import replace
    wr = replace(w, seed=w.seed + rank)
    host = workload_inputs(wr)
    set_bytes = w.io_bytes
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    R = max(2, math.ceil(3 * l2 / set_bytes))
    sets = []
    for r in range(R):
        q, k, v, rpb = (t.to(dev) for t in host)
        sets.append((q, k, v, rpb, torch.empty_like(q)))

    def step(i):
        q, k, v, rpb, out = sets[i % R]
        na2d.forward(q, k, v, rpb, w.ks, out=out)

    stream = torch.cuda.current_stream(dev)
    for i in range(max(args.warmup, 0)):
        step(i)
    torch.cuda.synchronize(dev)
    if na2d.device_status() != na2d.NA_OK:
        raise SystemExit("device status not OK after warm-up")

    # graphs of G steps (+ one for the remainder) so launches are back to back
    G = max(1, min(args.graph_steps, args.steps))
    n_full, rem = divmod(args.steps, G)

    def capture(n, offset):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(n):
                step(offset + i)
        return g

    g_full = capture(G, 0) if n_full else None
    g_rem = capture(rem, 0) if rem else None
    if g_full is not None:
        g_full.replay()  # one untimed replay of the captured graph
    torch.cuda.synchronize(dev)

    sampler = ClockSampler(local_rank) if rank == 0 else None
    if sampler:
        sampler.start()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(dev)
    torch.cuda.synchronize(dev)
    t_host0 = time.time()
    ev0.record(stream)
    for _ in range(n_full):
        g_full.replay()
    if g_rem is not None:
        g_rem.replay()
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    t_host1 = time.time()
    barrier(dev)
    local_ms = ev0.elapsed_time(ev1)
    total_ms = max_over_ranks(local_ms, dev)
    if sampler:
        sampler.mark(t_host0, t_host1)
    status = na2d.device_status()
    if status != na2d.NA_OK:
        raise SystemExit(f"device status {na2d.status_str(status)} after the timed region")

    # end to end through the host-buffer entry point (pinned buffers, copies timed)
    pin = [t.pin_memory() for t in host]
    out_host = torch.empty_like(host[0]).pin_memory()
    ws = torch.empty(na2d.host_workspace_bytes(*w.shape(), w.ks, host[0].dtype), dtype=torch.uint8, device=dev)
    for _ in range(3):
        na2d.forward_host(*pin, out_host, w.ks, ws)
    torch.cuda.synchronize(dev)
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
    peaks, peak_src = load_peaks()
    achieved_gbs = w.io_bytes / launch_s / 1e9
    tflops = w.flops / launch_s / 1e12
    traffic = profiled_traffic(kernel_source, w.name)
    roofline = {
        "bound": "hbm", "achieved": achieved_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
        "frac": achieved_gbs / peaks["hbm_gbs"], "traffic": traffic,
        "kernel": kernel_name, "launch_us": launch_s * 1e6, "peak_source": peak_src,
        "algorithmic_bytes": w.io_bytes,
        "tensor_view": {"achieved_tflops": tflops, "peak_tflops": peaks["bf16_tflops"],
                        "frac": tflops / peaks["bf16_tflops"]},
    }
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": workload_config(w, world, {
            "l2": f"rotating {R} input/output sets ({R * set_bytes / 1e6:.0f} MB, L2 {l2 / 1e6:.0f} MB)",
            "timing": f"CUDA graphs of {G} steps, CUDA events on the launching stream, max over ranks",
        }),
        "roofline": roofline,
        "e2e": {"value": e2e_value, "unit": UNIT,
                "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in host),
                "d2h_bytes_per_step": host[0].numel() * host[0].element_size(),
                "api": "na2d_forward_host", "steps": args.e2e_steps},
        "gpu_launches": args.steps,
    }
    if rank == 0:
        line["clocks"] = sampler.summary() if sampler else None
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_oracle_throughput(w, args.cpu_seconds)
        print(json.dumps(line), flush=True)
    del g_full, g_rem
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
