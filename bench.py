#!/usr/bin/env python
"""Benchmark of the frame-wise GDN scan (libgdn) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl libgdn|reference]

One step is one gdn_frame_scan over the whole 961-frame rollout (32 heads of
961 frames of 880 tokens, D = 64, bf16) with the inputs already resident in
HBM. The inputs (10.4 GB) are far larger than L2, so no L2 flush is needed
between steps. With N > 1 (torchrun) every rank scans its own copy of the
workload on its own GPU: the heads are independent, there is no collective on
the data path, and the scaling is weak. Rank 0 prints one JSON line.

After the timed region the same line gains, each timed with CUDA events on
the launching stream:
  step_latency   961 gdn_frame_step calls carrying the state in place (the
                 chunk-causal rollout), per-call p50/p99, and the final state's
                 distance to the scan's;
  workloads      the short clip and the stress batch through gdn_frame_scan,
                 and the causal temporal conv on the rollout's shapes, each with
                 its throughput and HBM roofline fraction;
  e2e            the headline through frame_scan_host on pinned host buffers;
  cpu_baseline   the float64 oracle on the host's cores.

--impl reference times the float64 CPU oracle (the only reference this
method has) on a bounded sample of the same workload, rank 0 only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from frame_wise_gated_scan_b200 import inputs  # noqa: E402

METRIC = "GDN frames·heads/s on the 961×880-token rollout (B=1, H=32, D=64, T=961, S=880, bf16)"
UNIT = "frames·heads/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="rollout", choices=sorted(inputs.WORKLOADS))
    ap.add_argument("--impl", default="libgdn", choices=["libgdn", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=2)
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="budget of the CPU-oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--frames", type=int, default=0,
                    help="run only the first N frames of the workload (profiling captures)")
    ap.add_argument("--step-calls", type=int, default=961,
                    help="gdn_frame_step calls timed one by one for the step latency (0: skip)")
    ap.add_argument("--no-stream", action="store_true",
                    help="skip the streaming-launch latency (a persistent kernel that waits for "
                         "host posts: never run it under a profiler's replay)")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the tiny, short, stress, conv and RoPE workloads (profiling captures)")
    ap.add_argument("--extra-steps", type=int, default=20,
                    help="timed launches of each extra workload")
    ap.add_argument("--extras", default="tiny,short,stress,conv,rope",
                    help="comma-separated extra workloads (tiny, short, stress, conv, rope)")
    ap.add_argument("--extra-frames", type=int, default=0,
                    help="cut the extra workloads to this many frames (profiling captures)")
    return ap.parse_args()


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


NOMINAL_HBM_GBS = 8000.0   # B200 HBM3e, the peak the GDN task quotes


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def roofline(alg_bytes, launch_s, traffic=None):
    """HBM roofline record for one launch of `alg_bytes` algorithmic bytes."""
    peak, kind = measured_peaks()
    achieved = alg_bytes / launch_s / 1e9
    return {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
            "frac": achieved / peak, "peak_kind": kind, "traffic": traffic,
            "frac_nominal": achieved / NOMINAL_HBM_GBS, "peak_nominal": NOMINAL_HBM_GBS,
            "algorithmic_bytes_per_launch": alg_bytes}


def _strip_comments(src: str) -> str:
    """C/C++ source without comments or blank lines, so that documentation
    edits do not count as kernel changes."""
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    return "\n".join(line.rstrip() for line in src.splitlines() if line.strip())


# Sources each timed scan kernel is built from (its own file, the PTX wrappers,
# the shared waits, the internal interface and the host helpers).
KERNEL_SOURCES = {
    "rollout": ("gdn_tc.cu", "sm100_ptx.h", "gdn_internal.h", "gdn_host.cu"),
    "short": ("gdn_tc.cu", "sm100_ptx.h", "gdn_internal.h", "gdn_host.cu"),
    "stress": ("gdn_tc128.cu", "sm100_ptx.h", "gdn_wait.cuh", "gdn_internal.h", "gdn_host.cu"),
}


def kernel_source_hash(workload: str) -> str:
    """SHA-256 of the code (comments removed) of the sources the workload's
    kernel is built from."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "frame_wise_gated_scan_b200", "csrc")
    for name in sorted(KERNEL_SOURCES.get(workload, ())):
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            h.update(name.encode() + b"\0" + _strip_comments(f.read()).encode())
    return h.hexdigest()


def recorded_traffic(workload: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel sources; else None."""
    path = os.path.join(ROOT, "profiles", f"scan_{workload}_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    if workload not in KERNEL_SOURCES or rec.get("source_sha256") != kernel_source_hash(workload):
        return None
    return rec.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region
    (read through a pipe; nothing is written to disk)."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.reader = None
        self.lines: list[str] = []

    def _drain(self):
        for line in self.proc.stdout:
            self.lines.append(line)

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.reader = threading.Thread(target=self._drain, daemon=True)
            self.reader.start()
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.reader.join(timeout=5)

    def summary(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        for line in list(self.lines):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9 and parts[1].replace(".", "").isdigit():
                rows.append(parts)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows]
        mx = max(float(r[2]) for r in rows)
        loaded = [float(r[1]) for r in rows if float(r[3]) > 200.0] or sm
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx, "reasons": reasons,
                "samples": len(rows), "power_w_max": max(float(r[3]) for r in rows)}


def _oracle_head_job(args):
    """One head of the workload through the float64 oracle (pool worker)."""
    wl, b, h, T = args
    from oracle import gdn_scan_ref
    q, k, v, g, be = inputs.head(wl, b, h, T)
    t0 = time.perf_counter()
    gdn_scan_ref(q, k, v, g, be)
    return time.perf_counter() - t0


def cpu_baseline(wl, seconds: float):
    """The float64 oracle, as it stands, on the host's cores: heads of the
    workload run in parallel, one per process of a spawn-started pool of
    os.cpu_count() processes, each over the first frames of its head, until
    about `seconds` of wall time is spent. Each process runs BLAS single-threaded
    (OMP/OPENBLAS/MKL_NUM_THREADS=1), so the cores go to heads, not to small
    matrix products."""
    import multiprocessing as mp
    cores = os.cpu_count() or 1
    chunk = min(wl.T, 24)
    env_keys = ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS")
    saved = {k: os.environ.get(k) for k in env_keys}
    for k in env_keys:
        os.environ[k] = "1"
    try:
        ctx = mp.get_context("spawn")
        with ctx.Pool(cores) as pool:
            pool.map(_oracle_head_job, [(wl, 0, 0, 1)] * cores)      # start-up, imports
            heads_done, oracle_s, t0 = 0, 0.0, time.perf_counter()
            while True:
                batch = [(wl, (i // wl.H) % wl.B, i % wl.H, chunk)
                         for i in range(heads_done, heads_done + cores)]
                oracle_s += sum(pool.map(_oracle_head_job, batch))
                heads_done += cores
                if time.perf_counter() - t0 >= seconds:
                    break
            wall = time.perf_counter() - t0
    finally:
        for k, v in saved.items():
            if v is None:
                os.environ.pop(k, None)
            else:
                os.environ[k] = v
    frames = heads_done * chunk
    # Each process times its oracle calls alone (its inputs are drawn outside
    # that time); all cores run heads at once, so the rate is frames over the
    # oracle time per core.
    return {"value": frames / (oracle_s / cores), "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{heads_done} head runs of the float64 oracle over the first {chunk} frames "
                      f"of a head (S={wl.S}, D={wl.D}), {cores} at a time in a pool of {cores} "
                      f"processes, BLAS single-threaded; {oracle_s:.1f} s of oracle time over "
                      f"{wall:.1f} s of wall time"}


def run_reference(args, wl):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    # each step: the oracle over one head for a bounded number of frames
    T = min(wl.T, 24)
    from oracle import gdn_scan_ref
    per_step = []
    for i in range(args.warmup + args.steps):
        h = i % wl.H
        q, k, v, g, be = inputs.head(wl, 0, h, T)
        t0 = time.perf_counter()
        gdn_scan_ref(q, k, v, g, be)
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            per_step.append(dt)
    total = sum(per_step)
    value = args.steps * T / total
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        cores = 1
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded, workload shapes)",
        "config": {"workload": wl.name, "B": wl.B, "H": wl.H, "D": wl.D, "T": wl.T, "S": wl.S,
                   "step": f"float64 oracle over {T} frames of one head"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"{args.steps} steps of {T} frames of one head (S={wl.S}, D={wl.D})"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def _time_launches(fn, n, stream, warmup=3):
    """Mean device time of `fn` (one launch each), CUDA events on `stream`."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(n):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / 1e3 / n


KERNEL_NAMES = {1: "simt", 2: "tcgen05", 3: "tcgen05 row-split (single frame)"}


def scan_workload(name, device, stream, n, frames=0):
    """One extra GDN workload through gdn_frame_scan: throughput and roofline."""
    import torch
    from frame_wise_gated_scan_b200 import gdn
    wl = inputs.WORKLOADS[name]
    if frames:
        wl = wl.with_(T=min(frames, wl.T))
    q, k, v, g, be = inputs.device_draw(wl, device)
    out = torch.empty_like(q)
    st = torch.empty((wl.B, wl.H, wl.D, wl.D), dtype=torch.float32, device=device)
    launch_s = _time_launches(lambda: gdn.frame_scan(q, k, v, g, be, None, out=out, state_out=st),
                              n, stream)
    if gdn.device_status() != 0:
        raise RuntimeError(f"a device-side wait ran out in the {name} workload")
    kern, ctas = gdn.plan(wl.B, wl.H, wl.T, wl.S, wl.D)
    rec = {"config": {"B": wl.B, "H": wl.H, "D": wl.D, "T": wl.T, "S": wl.S},
           "kernel": KERNEL_NAMES[kern], "ctas_per_head": ctas, "launches": n,
           "ms_per_launch": launch_s * 1e3, "value": wl.heads * wl.T / launch_s, "unit": UNIT,
           "gflops": inputs.flops(wl) / launch_s / 1e9,
           "roofline": roofline(inputs.algorithmic_bytes(wl), launch_s, recorded_traffic(name)),
           "l2": ("inputs larger than L2, no flush" if 3 * q.numel() * q.element_size() > 126e6
                  else "inputs fit in L2: launches run warm, back to back")}
    del q, k, v, out
    return rec


def conv_workload(device, stream, n, frames=0):
    """The causal temporal conv on the rollout's shapes: throughput and roofline."""
    import torch
    from frame_wise_gated_scan_b200 import gdn
    wl = inputs.CONV_WORKLOADS["conv_rollout"]
    if frames:
        wl = wl.with_(T=min(frames, wl.T))
    x, w, bias, cache = inputs.conv_device_draw(wl, device)
    y = torch.empty_like(x)
    c_out = torch.empty_like(cache)
    launch_s = _time_launches(
        lambda: gdn.temporal_conv(x, w, bias, cache, frames_per_block=wl.F, y=y, cache_out=c_out),
        n, stream)
    rec = {"config": {"B": wl.B, "T": wl.T, "S": wl.S, "C": wl.C, "frames_per_block": wl.F},
           "kernel": "cuda cores, 16-byte streams", "launches": n,
           "ms_per_launch": launch_s * 1e3,
           "value": wl.B * wl.T * wl.S / launch_s, "unit": "tokens/s",
           "roofline": roofline(inputs.conv_bytes(wl), launch_s),
           "l2": "inputs larger than L2 (3.5 GB read per launch), no flush"}
    del x, y
    return rec


def rope_workload(device, stream, n, frames=0):
    """3D RoPE of the rollout's queries (gdn_rope3d, out of place)."""
    import torch
    from frame_wise_gated_scan_b200 import gdn
    wl = inputs.WORKLOADS["rollout"]
    if frames:
        wl = wl.with_(T=min(frames, wl.T))
    q = inputs.device_draw(wl, device, seed_offset=7)[0]
    y = torch.empty_like(q)
    launch_s = _time_launches(lambda: gdn.rope3d(q, 40, 0, out=y), n, stream)
    nbytes = 2 * q.numel() * q.element_size()
    rec = {"config": {"B": wl.B, "H": wl.H, "D": wl.D, "T": wl.T, "S": wl.S, "grid_w": 40},
           "kernel": "cuda cores, 16-byte streams", "launches": n,
           "ms_per_launch": launch_s * 1e3,
           "value": wl.heads * wl.T * wl.S / launch_s, "unit": "token-rows/s",
           "roofline": roofline(nbytes, launch_s),
           "l2": "inputs larger than L2 (3.5 GB read per launch), no flush"}
    del q, y
    return rec


def main():
    args = parse()
    wl = inputs.WORKLOADS[args.workload]
    if wl.name == "step":
        wl = inputs.WORKLOADS["rollout"]
    if args.frames:
        wl = wl.with_(T=min(args.frames, wl.T))
    if args.impl == "reference":
        run_reference(args, wl)
        return
    import torch
    import torch.distributed as dist
    from frame_wise_gated_scan_b200 import gdn, multi

    rank, world, local = dist_env()
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", init_method="env://",
                                timeout=__import__("datetime").timedelta(seconds=300))
    device = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(device)

    kern, ctas = gdn.plan(wl.B, wl.H, wl.T, wl.S, wl.D)
    q, k, v, g, be = inputs.device_draw(wl, device)
    out = torch.empty_like(q)
    st = torch.empty((wl.B, wl.H, wl.D, wl.D), dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream(device)

    def step():
        gdn.frame_scan(q, k, v, g, be, None, out=out, state_out=st)

    # Warm-up: at least `warmup` steps (3 or more), and at least half a second
    # of them, so that clocks have settled before the timed steps.
    t_w = time.perf_counter()
    n_w = 0
    while n_w < max(3, args.warmup) or time.perf_counter() - t_w < 0.5:
        step()
        n_w += 1
        if n_w % 8 == 0:
            torch.cuda.synchronize(device)
    torch.cuda.synchronize(device)
    if gdn.device_status() != 0:
        raise RuntimeError("a device-side wait ran out during warm-up")

    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    launch_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                 for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(device)
    with ClockSampler(device.index if device.index is not None else 0) as clocks:
        ev0.record(stream)
        for i in range(args.steps):
            launch_ev[i][0].record(stream)
            step()
            launch_ev[i][1].record(stream)
        ev1.record(stream)
        torch.cuda.synchronize(device)
    if world > 1:
        dist.barrier()
    elapsed_ms = ev0.elapsed_time(ev1)
    launch_ms = [a.elapsed_time(b) for a, b in launch_ev]
    if gdn.device_status() != 0:
        raise RuntimeError("a device-side wait ran out during the timed steps")
    max_ms = multi.max_over_ranks(elapsed_ms, device)

    units = wl.heads * wl.T
    value = multi.whole_job_rate(units, args.steps, world, max_ms)
    mean_launch_s = statistics.mean(launch_ms) / 1e3
    alg_bytes = inputs.algorithmic_bytes(wl)
    roof = roofline(alg_bytes, mean_launch_s, recorded_traffic(wl.name))

    # Chunk-causal rollout: one gdn_frame_step per frame with the state carried
    # in place (the "step" workload), per-call latency, and the final state
    # against the scan's over the same frames.
    step_lat = None
    if args.step_calls > 0:
        n = min(args.step_calls, wl.T)
        frames = [tuple(x[:, :, t].contiguous() for x in (q, k, v, g, be)) for t in range(n)]
        o_step = torch.empty((wl.B, wl.H, wl.S, wl.D), dtype=q.dtype, device=device)
        s_step = torch.zeros((wl.B, wl.H, wl.D, wl.D), dtype=torch.float32, device=device)
        step_kern, step_ctas = gdn.plan(wl.B, wl.H, 1, wl.S, wl.D)
        for t in range(min(3, n)):
            gdn.frame_step(*frames[t], s_step, out=o_step, state_out=s_step)
        torch.cuda.synchronize(device)
        s_step.zero_()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(n)]
        # Device time per call: a short spin kernel ahead of the first event
        # keeps the GPU busy while the host enqueues the call, so the event
        # pair brackets the launch and the kernel, not the host's work.
        spin_cycles = int(80e-6 * 2.0e9)
        for t in range(n):
            torch.cuda._sleep(spin_cycles)
            evs[t][0].record(stream)
            gdn.frame_step(*frames[t], s_step, out=o_step, state_out=s_step)
            evs[t][1].record(stream)
            torch.cuda.synchronize(device)
        # Host time per call: the call plus a synchronize, wall clock.
        s_step.zero_()
        torch.cuda.synchronize(device)
        host_us = []
        for t in range(n):
            h0 = time.perf_counter()
            gdn.frame_step(*frames[t], s_step, out=o_step, state_out=s_step)
            torch.cuda.synchronize(device)
            host_us.append((time.perf_counter() - h0) * 1e6)
        if gdn.device_status() != 0:
            raise RuntimeError("a device-side wait ran out during the step calls")
        dev_us = sorted(a.elapsed_time(b) * 1e3 for a, b in evs)
        host_us.sort()
        pct = lambda xs, p: xs[min(len(xs) - 1, int(round(p / 100 * (len(xs) - 1))))]
        # the same frames back to back, no host round trip between calls
        s_step.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for t in range(n):
            gdn.frame_step(*frames[t], s_step, out=o_step, state_out=s_step)
        e1.record(stream)
        torch.cuda.synchronize(device)
        b2b_us = e0.elapsed_time(e1) * 1e3 / n
        state_vs_scan = None
        if n == wl.T:
            state_vs_scan = float((s_step - st).norm() / st.norm())
        # the same chain captured once as a CUDA graph and replayed: device time
        # per step without the host's per-call work
        s_step.zero_()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for t in range(n):
                gdn.frame_step(*frames[t], s_step, out=o_step, state_out=s_step)
        graph.replay()
        torch.cuda.synchronize(device)
        s_step.zero_()
        e0.record(stream)
        graph.replay()
        e1.record(stream)
        torch.cuda.synchronize(device)
        graph_us = e0.elapsed_time(e1) * 1e3 / n
        # The same graph replayed again: the mean time per step of each replay,
        # over 20 replays (consecutive steps keep their launch overlap).
        replay_us = []
        for _ in range(20):
            s_step.zero_()
            e0.record(stream)
            graph.replay()
            e1.record(stream)
            torch.cuda.synchronize(device)
            replay_us.append(e0.elapsed_time(e1) * 1e3 / n)
        replay_us.sort()
        del graph
        # Per-step device time inside a replayed graph: event records captured
        # between the steps (no host work, no configuration switch between
        # consecutive kernels).
        graph_steps = None
        try:
            # external: captured as event record nodes of the graph
            gev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(n + 1)]
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                gev[0].record()
                for t in range(n):
                    gdn.frame_step(*frames[t], s_step, out=o_step, state_out=s_step)
                    gev[t + 1].record()
            for _ in range(2):
                s_step.zero_()
                graph.replay()
                torch.cuda.synchronize(device)
            graph_steps = sorted(gev[t].elapsed_time(gev[t + 1]) * 1e3 for t in range(n))
            del graph
        except RuntimeError:
            graph_steps = None
        step_bytes = inputs.algorithmic_bytes(wl, 1) + wl.heads * wl.D * wl.D * 4
        step_lat = {"calls": n, "unit": "us",
                    "device_p50": pct(dev_us, 50), "device_p99": pct(dev_us, 99),
                    "host_p50": pct(host_us, 50), "host_p99": pct(host_us, 99),
                    "back_to_back_us_per_call": b2b_us,
                    "graph_us_per_step": graph_us,
                    "graph_replays_us_per_step_p50": pct(replay_us, 50),
                    "graph_replays_us_per_step_p99": pct(replay_us, 99),
                    "graph_step_p50": pct(graph_steps, 50) if graph_steps else None,
                    "graph_step_p99": pct(graph_steps, 99) if graph_steps else None,
                    # q, k, v read, out written, gates, the state read and written
                    "bytes_per_call": step_bytes,
                    "roofline_p50": roofline(
                        step_bytes, (pct(graph_steps, 50) if graph_steps else pct(dev_us, 50)) / 1e6),
                    # chained steps: the mean device time per step of the replayed graph
                    "roofline_graph": roofline(step_bytes, graph_us / 1e6),
                    "final_state_rel_diff_vs_scan": state_vs_scan,
                    "kernel": KERNEL_NAMES[step_kern], "ctas_per_head": step_ctas,
                    "how": "device: CUDA events around each call on its stream, the GPU kept "
                           "busy by a spin kernel while the host enqueues the call; graph_step: "
                           "events between consecutive steps inside a replayed CUDA graph, "
                           "which removes the overlap of consecutive launches (roofline_p50 "
                           "uses its p50); graph_us_per_step: one event pair around a replay "
                           "of the whole chain, divided by its steps; graph_replays: the same "
                           "over 20 more replays, p50 and p99 of the per-replay means; host: "
                           "call plus synchronize, wall clock; back to back: one event pair "
                           "around all calls"}
        del frames

    # The same rollout through the frame queue: one persistent launch, frames
    # posted one at a time by the host, each timed from post to done.
    stream_lat = None
    if args.step_calls > 0 and not args.no_stream:
        n = min(args.step_calls, wl.T)
        ring = lambda x: x[:, :, :n].permute(2, 0, 1, *range(3, x.dim())).contiguous()
        rings = [ring(x) for x in (q, k, v, g, be)]
        fs = gdn.FrameStream(*rings)
        lat = []
        for t in range(n):
            h0 = time.perf_counter()
            fs.post()
            fs.wait(t + 1)
            lat.append((time.perf_counter() - h0) * 1e6)
        s_stream = fs.close()
        lat.sort()
        pct = lambda xs, p: xs[min(len(xs) - 1, int(round(p / 100 * (len(xs) - 1))))]
        stream_lat = {"frames": n, "unit": "us", "p50": pct(lat, 50), "p99": pct(lat, 99),
                      "final_state_rel_diff_vs_scan":
                          float((s_stream - st).norm() / st.norm()) if n == wl.T else None,
                      "how": "one gdn_frame_stream launch over the rollout staged as a ring of "
                             "frame slots; the host posts frame t and polls for it to be done "
                             "(pinned-memory counters), wall clock per frame"}
        del rings, fs

    extras = None
    if not args.no_extras and rank == 0:
        want = [x.strip() for x in args.extras.split(",") if x.strip()]
        ef = args.extra_frames
        run = {"tiny": lambda: scan_workload("tiny", device, stream, args.extra_steps * 10, ef),
               "short": lambda: scan_workload("short", device, stream, args.extra_steps * 10, ef),
               "stress": lambda: scan_workload("stress", device, stream, args.extra_steps, ef),
               "conv": lambda: conv_workload(device, stream, args.extra_steps, ef),
               "rope": lambda: rope_workload(device, stream, args.extra_steps, ef)}
        extras = {name: run[name]() for name in want}

    # End to end through the public API on pinned host buffers.
    e2e = None
    if args.e2e_steps > 0:
        hq, hk, hv, hg, hb = (x.cpu().pin_memory() for x in (q, k, v, g, be))
        del q, k, v
        torch.cuda.empty_cache()
        staging = {}
        out_h = torch.empty(hq.shape, dtype=hq.dtype, pin_memory=True)
        st_h = torch.empty(st.shape, dtype=torch.float32, pin_memory=True)
        gdn.frame_scan_host(hq, hk, hv, hg, hb, staging=staging, out_host=out_h, state_host=st_h)
        if world > 1:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.e2e_steps):
            gdn.frame_scan_host(hq, hk, hv, hg, hb, staging=staging, out_host=out_h,
                                state_host=st_h)
        e1.record(stream)
        torch.cuda.synchronize(device)
        e2e_ms = multi.max_over_ranks(e0.elapsed_time(e1), device)
        h2d = sum(x.numel() * x.element_size() for x in (hq, hk, hv, hg, hb))
        d2h = out_h.numel() * out_h.element_size() + st_h.numel() * 4
        e2e = {"value": multi.whole_job_rate(units, args.e2e_steps, world, e2e_ms), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "steps": args.e2e_steps}

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    clock_rec = clocks.summary()
    if clock_rec.get("sm_mhz"):
        # time x clock, to compare runs on boxes whose clocks differ
        clock_rec["ms_per_step_x_sm_ghz"] = max_ms / args.steps * clock_rec["sm_mhz"] / 1e3
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "warmup_steps_run": n_w, "ms_per_step": max_ms / args.steps,
        "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded on the device; rollout recipe: Q,V ~ N(0,1), K rows "
                "L2-normalised, gamma ~ U(.95,1), beta ~ U(.2,1))",
        "config": {"workload": wl.name, "B": wl.B, "H": wl.H, "D": wl.D, "T": wl.T, "S": wl.S,
                   "global_batch": wl.B * world, "seq_len": wl.T * wl.S,
                   "parallelism": f"replicas x{world} (heads independent, no collective)",
                   "kernel": KERNEL_NAMES[kern], "ctas_per_head": ctas,
                   "l2": "inputs larger than L2 (10.4 GB read per step), no flush"},
        "gpu_launches": args.steps,
        "hbm_gbs": roof["achieved"],
        "roofline": roof,
        "clocks": clock_rec,
        "e2e": e2e,
        "step_latency": step_lat,
        "stream_latency": stream_lat,
        "workloads": extras,
    }
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl, args.cpu_seconds)
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
