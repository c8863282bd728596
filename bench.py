"""Benchmark: Newton-solved state elements per second on B200 (one JSON line).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--leg WORKLOAD:PART] [--skip-extras]

A step is one Newton (DEER) forward solve of the whole workload to convergence:
the fused cell + Jacobian + scan kernel iterating on the device until
max|delta| < tol.  Default workload: the DEER GRU benchmark shape (batch 16,
2^20 steps, state size 1, input width 2), synthetic seeded inputs.

Besides the headline, the line carries ``per_config``: every other workload of the
path timed on the device (CUDA events, L2 flushed between repeats, median), leg by
leg -- the projection GEMM, the Newton forward, the adjoint backward, the
projection backward and the two backward passes in one call (grad_xproj handed over
in bf16) of the LLM-width ParaGRU / ParaLSTM layers; the tanh RNN with
full DEER and quasi-DEER at n = 8 and 64, and the standalone dense linear scan at the
n = 64 shape -- each with its algorithmic bytes or flops
and its fraction of the bound it sits on, next to the fp64 oracle's sequential
rollout (the "naive sequential application") on all host cores and on one core.

``--leg WORKLOAD:PART`` times one leg alone and prints its line (profiling runs).

Multi-GPU (torchrun, one process per GPU): every rank solves its own batch of the
same shape (independent sequences, seed offset by rank); no collective on the
data path ("scaling": "weak"); the step time is the max over ranks.

--impl reference times the fp64 CPU oracle on the host cores, on rank 0 only: the
sequential rollout h_t = f(h_{t-1}, x_t) of the whole workload per step (the states
the Newton solve converges to), with the oracle's own Newton solve timed beside it.
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
KERNEL_NAME = "newton_staged_kernel<GruCell, TmaLong<GruCell, 2, 16, 256, 64>, 2, 256, 2>"


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


def _oracle_threads():
    return len(os.sched_getaffinity(0))


def _oracle_sample_model(w, inp, nb, units):
    """fp64 oracle model of a sample of the workload: the first ``nb`` sequences and, for
    the layers, the first ``units`` units (every sequence of the method is independent
    of the others, so a sample is a set of whole sequences)."""
    import oracle
    x = inp["x"][:nb]
    h0 = inp["h0"][:nb]
    if w.cell == wl.TANH or units >= w.H:
        sub = dict(inp, x=x, h0=h0)
        return oracle.model_from_inputs(w.cell, sub, quasi=w.quasi), h0, nb * (1 if w.cell == wl.TANH else w.H)
    H = w.H
    rows = np.concatenate([np.arange(g * H, g * H + units) for g in range(3)])
    xp = oracle.input_proj(x, inp["W"][rows], inp["bias"][rows]).reshape(nb, w.T, 3, units)
    m = oracle.Model(w.cell, xp, a=inp["a"][:, :units],
                     peep=inp["peep"][:, :units] if w.cell == wl.LSTM else None)
    return m, np.ascontiguousarray(h0[:, :units]), nb * units


def _time_cpu(fn, budget_s):
    """Mean wall time of fn() over as many runs as fit in about budget_s (at least one)."""
    fn()  # first touch of the sample's memory, page faults, thread start-up
    t0 = time.perf_counter()
    reps = 0
    while True:
        fn()
        reps += 1
        el = time.perf_counter() - t0
        if el > budget_s or reps >= 20:
            return el / reps, reps


def cpu_rollout(w, inp, nb, units, threads, budget_s=1.0):
    """The fp64 oracle's sequential rollout h_t = f(h_{t-1}, x_t) (the "naive
    sequential application" the pages' speedups are quoted against) on a sample of
    whole sequences, with ``threads`` OpenMP threads over independent sequences."""
    import oracle
    m, h0, _ = _oracle_sample_model(w, inp, nb, units)
    oracle.set_threads(threads)
    dt, reps = _time_cpu(lambda: m.rollout(h0), budget_s)
    if w.cell == wl.TANH:
        elems, what = nb * w.T * w.H, f"{nb} sequence(s) of {w.T} steps at state size {w.H}"
    else:
        elems, what = nb * w.T * units, f"{nb * units} unit sequence(s) of {w.T} steps ({nb} batch x {units} unit(s))"
    return {"value": elems / dt, "unit": "state elements/s", "cores": threads, "kind": "oracle",
            "sample": f"fp64 oracle sequential rollout of {what}, mean of {reps} run(s)"}


def _rollout_sample(w, steps, min_seq=1):
    """(batch rows, units) of a sample of whole sequences, about ``steps`` sequence steps
    (scaled by the n^2 cost of a dense step for the tanh RNN), at least ``min_seq``
    sequences where the workload has that many."""
    if w.cell == wl.TANH:
        return min(w.B, max(min_seq, steps * 64 // (w.H * w.H) // w.T)), w.H
    nseq = max(min_seq, steps // w.T)
    if nseq >= w.B:
        return w.B, min(w.H, nseq // w.B)
    return nseq, 1


def cpu_baselines(w, inp):
    """Rollout on all cores and on one core, each on a bounded sample."""
    threads = _oracle_threads()
    nb, units = _rollout_sample(w, 1 << 22, min_seq=threads)
    allc = cpu_rollout(w, inp, nb, units, threads)
    nb1, units1 = _rollout_sample(w, 1 << 20)
    one = cpu_rollout(w, inp, nb1, units1, 1, budget_s=0.5)
    return allc, one


def cpu_newton(w, inp, threads, budget_s=3.0):
    """The fp64 oracle's own Newton solve of the whole workload (for information)."""
    import oracle
    oracle.set_threads(threads)
    m = oracle.model_from_inputs(w.cell, inp, quasi=w.quasi)
    res = {}

    def run():
        res["it"] = m.newton(inp["h0"], max_iters=min(w.max_iters, 10_000), tol=w.tol)[1]

    dt, reps = _time_cpu(run, budget_s)
    return {"value": w.elems / dt, "unit": "state elements/s", "cores": threads, "kind": "oracle",
            "sample": f"fp64 oracle Newton solve of the whole workload ({res['it']} iterations), "
                      f"mean of {reps} run(s)"}


# ---------------------------------------------------------------- per-config legs
PER_CONFIG = ["gru_b1_t1024_in4_h8", "gru_b8_t4096_h2048_bf16", "lstm_b4_t8192_h1024_bf16",
              "tanh_b16_t65536_in4_n8_quasi", "tanh_b16_t65536_in4_n8_deer",
              "tanh_b16_t65536_in4_n64_deer", "tanh_b16_t65536_in4_n64_quasi"]
LAYER_PARTS = ["proj", "forward", "backward", "proj_backward", "layer_backward"]


def _fp32_peak_tflops():
    """FP32 FMA peak from the unit counts and the clock: 148 SMs x 128 FMA lanes x 2 flops
    x the maximum SM clock (MEASURED_PEAKS.json's sm_max_mhz, else 1965 MHz)."""
    mhz = 1965.0
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            mhz = float(json.load(f).get("sm_max_mhz", mhz))
    except Exception:
        pass
    return 148 * 128 * 2 * mhz * 1e6 / 1e12


def _bf16_peak_tflops():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]), "measured (burst)"
    except Exception:
        return 1590.0, "fallback"


def forward_bytes(w, iters, residual):
    """Algorithmic HBM bytes of one Newton forward solve: each iteration reads the inputs
    and the previous iterate once and writes the new one (the first reads no iterate, it
    is zero).  The residual at the result needs one more read of the inputs and states,
    except when the solve ran to its cap on a wide layer (H % 32 == 0, projected inputs):
    there the last iteration forms it from the inputs it already holds."""
    S, n = w.state_per_unit, w.H
    elems = w.B * w.T * w.H
    if w.cell == wl.TANH or (w.inp <= 8 and w.H <= 8):
        # raw inputs, projection recomputed in the kernel: x once per step per iteration
        xb = 4 * w.B * w.T * w.inp
        sb = 4 * elems * S
        per_first, per_next = xb + sb, xb + 2 * sb
        res = xb + sb
    else:
        pb = 4 * w.G * elems  # projected inputs, fp32
        sb = 4 * elems * S
        per_first, per_next = pb + sb, pb + 2 * sb
        res = pb + sb
    if iters <= 0:
        return 0
    if residual and w.H % 32 == 0 and not (w.inp <= 8 and w.H <= 8) and w.cell != wl.TANH and iters == w.max_iters:
        res = 0
    return per_first + (iters - 1) * per_next + (res if residual else 0)


def tanh_flops(w, iters, quasi):
    """Algorithmic fp32 flops of the tanh RNN forward: per step and iteration
    f = tanh(A h + U x + b) (2 n^2 + 2 n in), the Jacobian's scaling and the scan update
    (4 n); full DEER adds the chain products of the n x n Jacobians, n^3 multiply-adds
    per step, and the dense update n^2 (matrix-vector) instead of the diagonal one."""
    n = w.H
    per = 2 * n * n + 2 * n * w.inp + 4 * n
    if not quasi:
        per += 2 * n ** 3 + 2 * n * n
    return per * w.B * w.T * iters


class _Legs:
    """Device timing of the legs of one workload through the C ABI (inputs resident)."""

    def __init__(self, ctx, dev, stream, flush, reps, warmup):
        self.ctx, self.dev, self.stream, self.flush = ctx, dev, stream, flush
        self.reps, self.warmup = reps, warmup

    def time(self, fn):
        import torch
        for _ in range(self.warmup):
            fn()
        torch.cuda.synchronize(self.dev)
        ts = []
        for _ in range(self.reps):
            self.flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(self.stream)
            fn()
            b.record(self.stream)
            torch.cuda.synchronize(self.dev)
            ts.append(a.elapsed_time(b))
        return float(statistics.median(ts))


def _hbm_entry(ms, nbytes, peak):
    ach = nbytes / (ms / 1e3) / 1e9
    return {"bound": "hbm", "alg_bytes": int(nbytes), "achieved": ach, "peak": peak, "unit": "GB/s",
            "frac": ach / peak}


def _tensor_entry(ms, flops, peak, kind):
    ach = flops / (ms / 1e3) / 1e12
    return {"bound": "tensor", "alg_flops": int(flops), "achieved": ach, "peak": peak, "unit": "TFLOP/s",
            "frac": ach / peak, "peak_kind": kind}


def _alu_entry(ms, flops, peak):
    ach = flops / (ms / 1e3) / 1e12
    return {"bound": "alu", "alg_flops": int(flops), "achieved": ach, "peak": peak, "unit": "TFLOP/s",
            "frac": ach / peak, "peak_kind": "fp32 FMA: 148 SMs x 128 lanes x 2 flops x max SM clock"}


def measure_workload(L, w, inp, parts=None):
    """Time the legs of workload ``w``; returns {part: entry}."""
    import torch

    from nonlinear_rnn_solve_b200 import solve

    ctx, dev = L.ctx, L.dev
    hbm, _ = _peaks()
    out = {}
    f32 = lambda k: torch.from_numpy(inp[k]).to(dev)  # noqa: E731
    sc = {"iters": torch.zeros(1, dtype=torch.int32, device=dev), "delta": torch.zeros(1, device=dev),
          "residual": torch.zeros(1, device=dev)}
    elems = w.elems
    if w.cell == wl.TANH or (w.inp <= 8 and w.H <= 8):
        t = {k: f32(k) for k in inp if k != "g"}
        cell = ("tanh_quasi" if w.quasi else "tanh") if w.cell == wl.TANH else w.cell
        h_out = torch.empty(solve.state_shape(cell, w.B, w.T, w.H), device=dev)
        kw = dict(x=t["x"], W=t["W"], bias=t["bias"], A=t.get("A"), a=t.get("a"), peep=t.get("peep"))
        if w.cell == wl.TANH and not w.quasi and w.H == 8:
            # full DEER at n = 8 from h = 0 overflows in its first update on this input, in
            # the fp64 oracle as on the device: record that, nothing to time
            solve.newton_forward(ctx.ctx, cell, w.B, w.T, w.H, h0=t["h0"], max_iters=4, tol=w.tol,
                                 h_out=h_out, scalars=sc, **kw)
            torch.cuda.synchronize(dev)
            st = _ctx_status(ctx)
            return {"forward": {"diverges_from_zero_guess": True, "iters": int(sc["iters"].item()),
                                "device_status": st}}
        if w.cell == wl.TANH and not w.quasi and w.H > 32 and (parts is None or "scan" in parts):
            # the standalone dense linear scan (pararnn_linear_scan, dense kind) at the
            # workload's shape: out_t = J_t out_{t-1} + b_t, J_t [n, n] of N(0, 0.81 / n)
            # entries and b_t of N(0, 1) drawn on the device (seeded)
            from nonlinear_rnn_solve_b200 import PARARNN_SCAN_DENSE, pararnn_linear_scan
            n = w.H
            gen = torch.Generator(device=dev)
            gen.manual_seed(7)
            J = torch.randn(w.B, w.T, n, n, device=dev, generator=gen).mul_(0.9 / n ** 0.5)
            bb = torch.randn(w.B, w.T, n, device=dev, generator=gen)
            out_s = torch.empty_like(bb)
            ms = L.time(lambda: pararnn_linear_scan(ctx.ctx, PARARNN_SCAN_DENSE, J, bb, None, out_s, w.B, w.T, n))
            steps = w.B * w.T
            # chain map 2 n^3 + its offset 2 n^2 per step, re-walk 2 n^2; J and b read twice
            fl = steps * (2 * n ** 3 + 4 * n * n)
            nb = steps * (2 * (n * n + n) + n) * 4
            out["scan"] = {"ms": ms, "shape": f"J [B{w.B}, T{w.T}, {n}, {n}], forward",
                           "device_status": _ctx_status(ctx), "roofline": _alu_entry(ms, fl, _fp32_peak_tflops()),
                           "roofline_other": _hbm_entry(ms, nb, hbm)}
            del J, bb, out_s
            if parts is not None and "forward" not in parts:
                return out
        fn = lambda: solve.newton_forward(ctx.ctx, cell, w.B, w.T, w.H, h0=t["h0"],  # noqa: E731
                                          max_iters=w.max_iters, tol=w.tol, h_out=h_out, scalars=sc, **kw)
        ms = L.time(fn)
        it = int(sc["iters"].item())
        e = {"ms": ms, "iters": it, "elems_per_s": elems / (ms / 1e3), "device_status": _ctx_status(ctx)}
        nb = forward_bytes(w, it, False)
        if w.cell == wl.TANH:
            fl = tanh_flops(w, it, w.quasi)
            if not w.quasi and w.H > 32:
                # chain products on the tensor cores as three TF32 products each: the fp32
                # work against a third of the TF32 peak (measured bf16 x the nominal 1/2)
                bf, how = _bf16_peak_tflops()
                e["roofline"] = _tensor_entry(ms, fl, bf * 0.5 / 3.0,
                                              f"tf32 / 3 (three-product split), tf32 = bf16 {how} x 1/2")
            else:
                e["roofline"] = _alu_entry(ms, fl, _fp32_peak_tflops()) if not w.quasi else _hbm_entry(ms, nb, hbm)
            e["roofline_other"] = _hbm_entry(ms, nb, hbm) if not w.quasi else _alu_entry(ms, fl, _fp32_peak_tflops())
        elif w.elems < 1 << 20:
            e["roofline"] = dict(_hbm_entry(ms, nb, hbm), bound="latency",
                                 note="8,192 state elements: launch and iteration latency, no bandwidth claim")
        else:
            e["roofline"] = _hbm_entry(ms, nb, hbm)
        out["forward"] = e
        if w.cell == wl.GRU:
            # ELK (damping 1) on the same shape: per-iteration algorithmic bytes as the
            # Newton solve's, over its own time; the ratio compares bytes/s
            lam = 1.0
            fe = lambda: solve.newton_forward(ctx.ctx, cell, w.B, w.T, w.H, h0=t["h0"],  # noqa: E731
                                              max_iters=w.max_iters, tol=w.tol, h_out=h_out, scalars=sc,
                                              solver="elk", damping=lam, **kw)
            ms_e = L.time(fe)
            it_e = int(sc["iters"].item())
            nb_e = forward_bytes(w, it_e, False)
            ee = {"ms": ms_e, "iters": it_e, "damping": lam, "device_status": _ctx_status(ctx)}
            ee["roofline"] = _hbm_entry(ms_e, nb_e, hbm)
            ee["bytes_per_s_vs_newton"] = (nb_e / ms_e) / (nb / ms)
            if w.H <= 8 and w.elems < 1 << 20:
                ee["roofline"] = dict(ee["roofline"], bound="latency",
                                      note="8,192 state elements: launch and iteration latency, no bandwidth claim")
            out["elk"] = ee
        return out
    # the LLM-width layers: projection GEMM, forward on xproj, adjoint, projection backward
    parts = parts or LAYER_PARTS
    B, T, H, K = w.B, w.T, w.H, w.inp
    M, N = B * T, 3 * H
    bf = lambda a: torch.from_numpy(wl.bf16_bits(a).view(np.int16)).to(dev).view(torch.bfloat16)  # noqa: E731
    x = bf(inp["x"].reshape(M, K))
    W = bf(inp["W"])
    bias = f32("bias")
    a = f32("a")
    peep = f32("peep") if w.cell == wl.LSTM else None
    h0 = f32("h0")
    xp = torch.empty(M, N, device=dev)
    from nonlinear_rnn_solve_b200 import pararnn_input_proj
    pararnn_input_proj(ctx.ctx, x, W, bias, xp)
    bf_peak, bf_kind = _bf16_peak_tflops()
    if "proj" in parts:
        ms = L.time(lambda: pararnn_input_proj(ctx.ctx, x, W, bias, xp))
        out["proj"] = {"ms": ms, "shape": f"M{M} K{K} N{N} bf16 -> fp32",
                       "roofline": _tensor_entry(ms, 2 * M * N * K, bf_peak, bf_kind)}
    xp4 = xp.view(B, T, 3, H)
    h = torch.empty(solve.state_shape(w.cell, B, T, H), device=dev)
    fwd = lambda: solve.newton_forward(ctx.ctx, w.cell, B, T, H, xproj=xp4, a=a, peep=peep,  # noqa: E731
                                       h0=h0, max_iters=w.max_iters, tol=w.tol, residual=w.residual,
                                       h_out=h, scalars=sc)
    if "forward" in parts:
        ms = L.time(fwd)
        it = int(sc["iters"].item())
        e = {"ms": ms, "iters": it, "elems_per_s": elems / (ms / 1e3), "device_status": _ctx_status(ctx)}
        if w.residual:
            e["residual"] = float(sc["residual"].item())
        e["roofline"] = _hbm_entry(ms, forward_bytes(w, it, w.residual), hbm)
        out["forward"] = e
    else:
        fwd()
    if "backward" in parts or "proj_backward" in parts or "layer_backward" in parts:
        g = f32("g")
        gx = torch.empty(B, T, 3, H, device=dev)
        gp = torch.empty(5 if w.cell == wl.LSTM else 3, H, device=dev)
        gh0 = torch.empty_like(h0)
        from nonlinear_rnn_solve_b200 import make_params, pararnn_adjoint_backward
        prm = make_params(solve.CELLS[w.cell], B, T, H, 0, a=a, peep=peep)
        bwd = lambda: pararnn_adjoint_backward(ctx.ctx, xp4, prm, h0, h, g, gx, gp, gh0)  # noqa: E731
        if "backward" in parts:
            ms = L.time(bwd)
            S = w.state_per_unit
            nb = elems * (4 * S + 12 + 4 * S + 12)  # states, xproj, upstream grad; grad_xproj
            out["backward"] = {"ms": ms, "elems_per_s": elems / (ms / 1e3), "device_status": _ctx_status(ctx),
                               "roofline": _hbm_entry(ms, nb, hbm)}
        else:
            bwd()
        if "layer_backward" in parts:
            # the same two passes in one call, grad_xproj handed from the adjoint to the
            # products in bf16 (no fp32 copy written or read)
            from nonlinear_rnn_solve_b200 import pararnn_layer_backward
            lx, lW, lb = torch.empty(M, K, device=dev), torch.empty(N, K, device=dev), torch.empty(N, device=dev)
            lp, lh0 = torch.empty_like(gp), torch.empty_like(h0)
            ms = L.time(lambda: pararnn_layer_backward(ctx.ctx, xp4, prm, h0, h, g, x, W, lx, lW, lb, lp, lh0))
            out["layer_backward"] = {"ms": ms, "device_status": _ctx_status(ctx),
                                     "shape": "adjoint + grad_x, grad_W, grad_bias in one call (bf16 grad_xproj)",
                                     "roofline": _tensor_entry(ms, 4 * M * N * K, bf_peak, bf_kind)}
            del lx, lW, lb, lp, lh0
        del g
        if "proj_backward" in parts:
            from nonlinear_rnn_solve_b200 import pararnn_input_proj_backward
            gxx = torch.empty(M, K, device=dev)
            gW = torch.empty(N, K, device=dev)
            gb = torch.empty(N, device=dev)
            gx2 = gx.view(M, N)
            ms = L.time(lambda: pararnn_input_proj_backward(ctx.ctx, gx2, x, W, gxx, gW, gb))
            out["proj_backward"] = {"ms": ms, "shape": f"grad_x [M{M}, K{K}] and grad_W [N{N}, K{K}] from "
                                                       f"fp32 grad_xproj (bf16 tensor-core products)",
                                    "roofline": _tensor_entry(ms, 4 * M * N * K, bf_peak, bf_kind)}
    return out


def _ctx_status(ctx):
    st = ctx.status()
    return int(st)


def per_config(ctx, dev, stream, flush, names=None, with_cpu=True):
    """Every non-headline workload, leg by leg, with the rollout baselines."""
    res = {}
    L = _Legs(ctx, dev, stream, flush, reps=5, warmup=3)
    for name in names or PER_CONFIG:
        w = wl.WORKLOADS[name]
        inp = wl.generate(w)
        t0 = time.perf_counter()
        r = {"shape": {"B": w.B, "T": w.T, "H": w.H, "in": w.inp, "tol": w.tol, "max_iters": w.max_iters}}
        try:
            r.update(measure_workload(L, w, inp))
        except Exception as e:  # a failing leg is reported, the others still run
            r["error"] = f"{type(e).__name__}: {e}"
        if with_cpu and not (w.cell == wl.TANH and not w.quasi and w.H == 8):
            allc, one = cpu_baselines(w, inp)
            r["cpu_rollout"] = allc
            r["cpu_rollout_1core"] = one
            fw = r.get("forward", {})
            if "elems_per_s" in fw:
                r["speedup_vs_rollout"] = fw["elems_per_s"] / allc["value"]
                r["speedup_vs_rollout_1core"] = fw["elems_per_s"] / one["value"]
        r["wall_s"] = time.perf_counter() - t0
        res[name] = r
        del inp
    return res


def run_leg(args):
    """Time one leg alone and print its line (the profiling runs use this)."""
    import torch

    from nonlinear_rnn_solve_b200 import Context
    name, _, part = args.leg.partition(":")
    w = wl.WORKLOADS[name]
    if args.leg_batch:
        w = w.resized(B=args.leg_batch)  # a smaller case of the same shape (ncu captures)
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    ctx = Context(0, stream)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    L = _Legs(ctx, dev, stream, flush, reps=args.steps, warmup=args.warmup)
    inp = wl.generate(w)
    r = measure_workload(L, w, inp, parts=[part] if part else None)
    print(json.dumps({"leg": args.leg, "steps": args.steps, "warmup": args.warmup, "result": r}), flush=True)
    ctx.close()


def run_reference(args, w):
    ws, rank, _ = _dist()
    if rank != 0:
        return
    inp = wl.generate(w)
    import oracle
    threads = _oracle_threads()
    oracle.set_threads(threads)
    m = oracle.model_from_inputs(w.cell, inp, quasi=w.quasi)
    for _ in range(args.warmup):
        m.rollout(inp["h0"])
    ts = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        m.rollout(inp["h0"])
        ts.append(time.perf_counter() - t0)
    ms = 1e3 * sum(ts) / len(ts)
    value = w.elems / (ms / 1e3)
    line = {"metric": METRIC, "value": value, "unit": "state elements/s", "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": w.name, "B": w.B, "T": w.T, "H": w.H, "in": w.inp, "tol": w.tol},
            "cpu_baseline": {"value": value, "unit": "state elements/s", "cores": threads, "kind": "oracle",
                             "sample": "whole workload per step: fp64 oracle sequential rollout "
                                       "h_t = f(h_{t-1}, x_t), OpenMP over independent sequences"},
            "oracle_newton": cpu_newton(w, inp, threads),
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

    sc = {"iters": torch.zeros(1, dtype=torch.int32, device=dev), "delta": torch.zeros(1, device=dev)}

    def step(h_out=None):
        return solve.newton_forward(ctx.ctx, w.cell, w.B, w.T, w.H, x=t["x"], W=t["W"], bias=t["bias"],
                                    a=t.get("a"), peep=t.get("peep"), h0=t["h0"], max_iters=w.max_iters,
                                    tol=w.tol, h_out=h_out, scalars=sc)

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
            allc, one = cpu_baselines(w, inp)
            line["cpu_baseline"] = dict(allc, one_core=one, oracle_newton=cpu_newton(w, inp, allc["cores"]))
            line["per_config"] = per_config(ctx, dev, stream, flush)
            if w.cell == wl.GRU:
                # ELK on the headline shape, its bytes/s against the Newton solve's
                line["elk_same_shape"] = measure_workload(_Legs(ctx, dev, stream, flush, reps=5, warmup=3), w,
                                                          inp).get("elk")
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
                    help="skip the e2e, CPU-baseline and per-config legs (for profiler runs)")
    ap.add_argument("--leg", default=None,
                    help="WORKLOAD[:PART]: time one leg alone (PART: proj, forward, backward, proj_backward, "
                         "layer_backward; scan for the n = 64 tanh DEER workload)")
    ap.add_argument("--leg-batch", type=int, default=0,
                    help="with --leg: the workload's batch replaced by this one (a smaller case for profiling)")
    args = ap.parse_args()
    w = wl.WORKLOADS[args.workload]
    if args.leg:
        run_leg(args)
    elif args.impl == "reference":
        run_reference(args, w)
    else:
        run_ours(args, w)


if __name__ == "__main__":
    main()
