"""Benchmark: Newton-solved state elements per second on B200 (one JSON line).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

A step is one Newton (DEER) forward solve of the whole workload to convergence:
the fused cell + Jacobian + scan kernel iterating on the device until
max|delta| < tol.  Default workload: the DEER GRU benchmark shape (batch 16,
2^20 steps, state size 1, input width 2), synthetic seeded inputs.

Multi-GPU (torchrun, one process per GPU): every rank solves its own batch of the
same shape (independent sequences, seed offset by rank); no collective on the
data path ("scaling": "weak"); the step time is the max over ranks.

--impl reference times the fp64 CPU oracle (the sequential-in-time Newton solve
as the pages describe it) on the host cores, on rank 0 only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from nonlinear_rnn_solve_b200 import workloads as wl  # noqa: E402

METRIC = "Newton-solved state elements/s (B*T*H/s) and % of HBM roofline"
# The DEER summary reports this exact workload (GRU, 1M steps, batch 16, n = 1) at
# 15 ms on a V100: 16 * 2^20 / 15 ms state elements per second (context only).
PUBLISHED_ELEMS_PER_S = {"gru_b16_t1048576_in2_h1": 16 * (1 << 20) / 15e-3}
# sources of the dominant kernel (the staged Newton kernel); a committed traffic figure
# applies only while they are unchanged
KERNEL_SOURCES = ["common.cuh", "cells.cuh", "newton_common.cuh", "staged_tiles.cuh", "newton_staged.cu"]
KERNEL_NAME = "newton_staged_kernel<GruCell, TmaLong<GruCell, 2, 16, 256, 256>, 2, 256, 2>"


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def _src_sha():
    h = hashlib.sha256()
    for n in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "nonlinear_rnn_solve_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def _traffic(workload):
    """DRAM bytes per launch from the committed ncu summary, if it matches the source."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(path):
        return None
    sha = _src_sha()
    for line in open(path):
        parts = line.split()
        if len(parts) == 4 and not line.startswith("#") and parts[0] == workload and parts[1] == sha:
            return float(parts[3])
    return None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.rows = []
        self._stop = threading.Event()
        self._t = None

    def _run(self):
        try:
            p = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                                  "--format=csv,noheader,nounits", "-lms", "100"],
                                 stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            return
        try:
            while not self._stop.is_set():
                line = p.stdout.readline()
                if not line:
                    break
                self.rows.append([x.strip() for x in line.split(",")])
        finally:
            p.terminate()
            try:
                p.wait(timeout=5)
            except Exception:
                p.kill()

    def __enter__(self):
        self._t = threading.Thread(target=self._run, daemon=True)
        self._t.start()
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        time.sleep(0.2)
        self._stop.set()
        self._t.join(timeout=10)

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in self.rows:
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
            except (ValueError, IndexError):
                continue
            for n, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def rank_workload(w, rank, world):
    """The workload one rank solves: same shape, its own independent sequences."""
    return w.resized(seed=w.seed + 1000 * rank) if world > 1 else w


def max_over_ranks(values, device=None):
    """Element-wise max of per-rank timings (the job's time is its slowest rank)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def _cpu_oracle_sample(w, inp, max_seconds=20.0):
    """Time the fp64 oracle Newton solve on a bounded sample of the workload."""
    import oracle
    threads = len(os.sched_getaffinity(0))
    oracle.set_threads(threads)
    # sample: whole sequences of the workload (every one has the same length)
    nb = w.B
    sub = {k: (v[:nb] if k in ("x", "h0", "g") else v) for k, v in inp.items()}
    m = oracle.model_from_inputs(w.cell, sub, quasi=w.quasi)
    t0 = time.perf_counter()
    reps = 0
    while True:
        _, iters, _ = m.newton(sub["h0"], max_iters=min(w.max_iters, 10_000), tol=w.tol)
        reps += 1
        if time.perf_counter() - t0 > max_seconds / 4 or reps >= 3:
            break
    dt = (time.perf_counter() - t0) / reps
    elems = nb * w.T * w.H
    return {"value": elems / dt, "unit": "state elements/s", "cores": threads, "kind": "oracle",
            "sample": f"fp64 oracle Newton solve of {nb} x {w.T} x {w.H} states ({iters} iterations), "
                      f"mean of {reps} run(s)"}


def run_reference(args, w):
    ws, rank, _ = _dist()
    if rank != 0:
        return
    inp = wl.generate(w)
    import oracle
    threads = len(os.sched_getaffinity(0))
    oracle.set_threads(threads)
    m = oracle.model_from_inputs(w.cell, inp, quasi=w.quasi)
    for _ in range(args.warmup):
        m.newton(inp["h0"], max_iters=w.max_iters, tol=w.tol)
    ts = []
    iters = 0
    for _ in range(args.steps):
        t0 = time.perf_counter()
        _, iters, _ = m.newton(inp["h0"], max_iters=w.max_iters, tol=w.tol)
        ts.append(time.perf_counter() - t0)
    ms = 1e3 * sum(ts) / len(ts)
    value = w.elems / (ms / 1e3)
    line = {"metric": METRIC, "value": value, "unit": "state elements/s", "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": w.name, "B": w.B, "T": w.T, "H": w.H, "in": w.inp, "iters": iters,
                       "tol": w.tol},
            "cpu_baseline": {"value": value, "unit": "state elements/s", "cores": threads, "kind": "oracle",
                             "sample": f"whole workload per step, fp64 oracle Newton solve ({iters} iterations)"},
            "e2e": {"value": value, "unit": "state elements/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def _e2e(args, w, ctx, inp, dev, stream, flush, h_out):
    """Same solve through the C ABI with host buffers: every step copies its inputs from
    pinned memory, solves, and reads its states back, all inside the timed region.
    Two CUDA streams take alternate steps, each with its own context, device buffers and
    pinned output, so a step's copies overlap its neighbour's solve (the way a stream of
    batches is served); the time is from the first step's start to the last step's end,
    divided by the steps."""
    import torch

    from nonlinear_rnn_solve_b200 import Context, solve

    host_in = {k: v.pin_memory() for k, v in ((k, torch.from_numpy(v)) for k, v in inp.items())}
    streams = [stream, torch.cuda.Stream(dev)]
    ctxs = [ctx, Context(dev.index, streams[1])]
    dev_in = [{k: torch.empty_like(v, device=dev) for k, v in host_in.items()} for _ in range(2)]
    h_outs = [h_out, torch.empty_like(h_out)]
    host_out = [torch.empty(h_out.shape, dtype=torch.float32).pin_memory() for _ in range(2)]
    h2d = sum(v.numel() * v.element_size() for v in host_in.values())
    d2h = host_out[0].numel() * 4

    def e2e_step(i, flush_l2):
        sl = i % 2
        with torch.cuda.stream(streams[sl]):
            if flush_l2:
                flush.zero_()
            for k in host_in:
                dev_in[sl][k].copy_(host_in[k], non_blocking=True)
            d = dev_in[sl]
            o = solve.newton_forward(ctxs[sl].ctx, w.cell, w.B, w.T, w.H, x=d["x"], W=d["W"], bias=d["bias"],
                                     a=d.get("a"), peep=d.get("peep"), h0=d["h0"], max_iters=w.max_iters,
                                     tol=w.tol, h_out=h_outs[sl])
            host_out[sl].copy_(o["h"], non_blocking=True)

    for i in range(4):
        e2e_step(i, False)
    torch.cuda.synchronize(dev)
    start = torch.cuda.Event(enable_timing=True)
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    start.record(streams[0])
    streams[1].wait_event(start)
    for i in range(args.steps):
        e2e_step(i, True)
    for sl in range(2):
        ends[sl].record(streams[sl])
    torch.cuda.synchronize(dev)
    e2e_ms = max(start.elapsed_time(e) for e in ends) / args.steps
    bad = ctxs[1].status()
    ctxs[1].close()
    if bad != 0:
        raise RuntimeError("device status of the second end-to-end stream: %d" % bad)
    return e2e_ms, h2d, d2h


def run_ours(args, w):
    import torch
    import torch.distributed as dist

    from nonlinear_rnn_solve_b200 import Context, pararnn_last_launch_count, solve

    ws, rank, local = _dist()
    if ws > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    dev = torch.device("cuda", local if ws > 1 else 0)
    torch.cuda.set_device(dev)
    inp = wl.generate(rank_workload(w, rank, ws))
    t = {k: torch.from_numpy(v).to(dev) for k, v in inp.items()}
    stream = torch.cuda.current_stream(dev)
    ctx = Context(dev.index, stream)

    def step(h_out=None):
        return solve.newton_forward(ctx.ctx, w.cell, w.B, w.T, w.H, x=t["x"], W=t["W"], bias=t["bias"],
                                    a=t.get("a"), peep=t.get("peep"), h0=t["h0"], max_iters=w.max_iters,
                                    tol=w.tol, h_out=h_out)

    h_out = torch.empty(solve.state_shape(w.cell, w.B, w.T, w.H), device=dev)
    for _ in range(max(args.warmup, 3)):
        out = step(h_out)
    torch.cuda.synchronize(dev)
    if ctx.status() != 0:
        raise RuntimeError("device status after warm-up: %d" % ctx.status())
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)  # > 126 MB L2
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    launches = 0
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(dev.index) as clk:
        wall0 = time.perf_counter()
        for i in range(args.steps):
            flush.zero_()
            evs[i][0].record(stream)
            out = step(h_out)
            evs[i][1].record(stream)
            launches += pararnn_last_launch_count(ctx.ctx)
        torch.cuda.synchronize(dev)
        wall = time.perf_counter() - wall0
    if ws > 1:
        dist.barrier()
    step_ms = [a.elapsed_time(b) for a, b in evs]
    ms = sum(step_ms) / len(step_ms)
    iters = int(out["iters"].item())
    status = ctx.status()

    # end to end through the C ABI with host buffers (see _e2e)
    if args.skip_extras:
        e2e_ms, h2d, d2h = float("nan"), 0, 0
    else:
        e2e_ms, h2d, d2h = _e2e(args, w, ctx, inp, dev, stream, flush, h_out)

    ms, e2e_ms = max_over_ranks([ms, e2e_ms], device=dev)
    units = w.elems * ws
    value = units / (ms / 1e3)
    peak, peak_kind = _peaks()
    per_elem = (12 + 16 * (iters - 1)) if iters > 0 else 0
    alg_bytes = w.elems * per_elem + 4 * (3 * w.H * (w.inp + 1) + 3 * w.H)
    achieved = alg_bytes / (ms / 1e3) / 1e9
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "state elements/s", "n_gpus": ws,
            "steps": args.steps, "warmup": max(args.warmup, 3), "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": (value / ws / PUBLISHED_ELEMS_PER_S[w.name]) if w.name in PUBLISHED_ELEMS_PER_S else None,
            "dtype": "f32", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "T": w.T, "H": w.H, "in": w.inp, "tol": w.tol,
                       "iters": iters, "l2": "flushed between steps (512 MiB write)",
                       "parallelism": f"independent batch per GPU x{ws}", "device_status": status},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": _traffic(w.name), "kernel": KERNEL_NAME,
                         "alg_bytes_per_launch": alg_bytes, "peak_source": peak_kind},
            "e2e": {"value": units / (e2e_ms / 1e3), "unit": "state elements/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                    "note": "host buffers; two streams take alternate steps (copies overlap the other step's solve)"},
            "gpu_launches": launches,
            "clocks": clk.summary(),
            "wall_s_timed": wall,
        }
        if ws == 1 and not args.skip_extras:
            line["cpu_baseline"] = _cpu_oracle_sample(w, inp)
        print(json.dumps(line), flush=True)
    ctx.close()
    if ws > 1:
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=wl.BENCH_WORKLOAD, choices=sorted(wl.WORKLOADS))
    ap.add_argument("--skip-extras", action="store_true",
                    help="skip the e2e and CPU-baseline legs (for profiler runs)")
    args = ap.parse_args()
    w = wl.WORKLOADS[args.workload]
    if args.impl == "reference":
        run_reference(args, w)
    else:
        run_ours(args, w)


if __name__ == "__main__":
    main()
