"""GPU parity: Newton (DEER) forward for ParaGRU and ParaLSTM against the fp64 oracle.

Bars: Newton iteration counts identical to the oracle's; converged states within
1e-4 (max abs); unconverged iterates (fixed iteration counts) within 1e-4 of the
oracle's iterate relative to max(1, |h|_max).  Inputs are the seeded workloads
(full sizes for the ParaGRU benchmark shapes, reduced ones elsewhere).
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import gpu, host, max_abs, need_gpu

from nonlinear_rnn_solve_b200 import (PARARNN_NOTCONVERGED, Context, pararnn_debug_set, solve)
from nonlinear_rnn_solve_b200 import workloads as wl

pytestmark = pytest.mark.gpu
TOL_STATE = 1e-4


@pytest.fixture(scope="module")
def ctx():
    need_gpu()
    c = Context(0)
    yield c
    c.close()


def _run_fused(ctx, w, inp, max_iters=None, tol=None, residual=False, delta_log=None):
    t = {k: gpu(v) for k, v in inp.items() if v is not None}
    if delta_log is not None:
        pararnn_debug_set(ctx.ctx, 3, delta_log.data_ptr())
        pararnn_debug_set(ctx.ctx, 4, delta_log.numel())
    out = solve.newton_forward(ctx.ctx, w.cell, w.B, w.T, w.H, x=t["x"], W=t["W"], bias=t["bias"],
                               a=t.get("a"), peep=t.get("peep"), h0=t["h0"],
                               max_iters=w.max_iters if max_iters is None else max_iters,
                               tol=w.tol if tol is None else tol, residual=residual)
    torch.cuda.synchronize()
    if delta_log is not None:
        pararnn_debug_set(ctx.ctx, 4, 0)
    return out


def _oracle_model(w, inp):
    # the oracle consumes the same inputs; its projection is fp64
    return oracle.model_from_inputs(w.cell, inp)


@pytest.mark.parametrize("name", ["gru_b1_t1024_in4_h8", "gru_b16_t1048576_in2_h1"])
def test_gru_workloads_full_size(ctx, name):
    w = wl.WORKLOADS[name]
    inp = wl.generate(w)
    log = torch.zeros(64, device="cuda:0")
    out = _run_fused(ctx, w, inp, delta_log=log)
    assert ctx.status() == 0
    m = _oracle_model(w, inp)
    h_ref, it_ref, d_ref = m.newton(inp["h0"], max_iters=min(w.max_iters, 64), tol=w.tol)
    it = int(out["iters"].item())
    d_gpu = host(log)[:it]
    assert it == it_ref, f"iterations {it} vs oracle {it_ref}; deltas gpu {d_gpu} oracle {d_ref}"
    assert max_abs(host(out["h"]), h_ref) <= TOL_STATE
    # delta trajectory agrees until it reaches the fp32 floor
    for k in range(it):
        assert abs(d_gpu[k] - d_ref[k]) <= 1e-4 * max(1.0, d_ref[k]) + 2e-6
    assert abs(float(out["delta"].item()) - d_gpu[-1]) == 0.0


SMALL = [  # (cell, B, T, H, in, seed)
    ("gru", 1, 1, 1, 2, 11),
    ("gru", 2, 37, 3, 3, 12),
    ("gru", 3, 5000, 5, 1, 13),
    ("gru", 2, 9000, 1, 2, 14),
    ("gru", 1, 700, 33, 4, 15),
    ("lstm", 1, 1, 1, 2, 16),
    ("lstm", 2, 777, 33, 4, 17),
    ("lstm", 1, 3001, 1, 2, 18),
    ("lstm", 2, 400, 8, 6, 19),
]


def _small_workload(cell, B, T, H, inp, seed):
    base = wl.WORKLOADS["gru_b1_t1024_in4_h8"] if cell == "gru" else wl.WORKLOADS["lstm_b4_t8192_h1024_bf16"]
    return base.resized(B=B, T=T, H=H, inp=inp, seed=seed, bf16=False, tol=1e-5 if cell == "lstm" else 1e-6,
                        max_iters=T + 1, w_dist="uniform_fan_in")


@pytest.mark.parametrize("case", SMALL)
def test_small_shapes_fused_projection(ctx, case):
    w = _small_workload(*case)
    inp = wl.generate(w)
    rng = np.random.default_rng(case[-1])
    inp["h0"] = (rng.standard_normal(inp["h0"].shape) * 0.5).astype(np.float32)
    out = _run_fused(ctx, w, inp, residual=True)
    assert ctx.status() == 0
    m = _oracle_model(w, inp)
    h_ref, it_ref, d_ref = m.newton(inp["h0"], max_iters=w.max_iters, tol=w.tol)
    assert int(out["iters"].item()) == it_ref, (int(out["iters"].item()), it_ref, d_ref)
    h = host(out["h"])
    assert max_abs(h, h_ref) <= TOL_STATE
    assert abs(float(out["residual"].item()) - m.residual(h, inp["h0"])) <= 2e-6


@pytest.mark.parametrize("cell,B,T,H", [("gru", 2, 1500, 40), ("gru", 1, 300, 2048), ("lstm", 2, 1000, 40),
                                        ("lstm", 1, 600, 96)])
def test_xproj_path_fixed_iterations(ctx, cell, B, T, H):
    """xproj given (as after the projection GEMM), tol = 0: exactly k iterations."""
    rng = np.random.default_rng(B * 7 + T + H)
    xp = (rng.standard_normal((B, T, 3, H)) * 0.8).astype(np.float32)
    a = rng.uniform(-0.9, 0.9, (3, H)).astype(np.float32)
    peep = rng.uniform(-0.5, 0.5, (2, H)).astype(np.float32) if cell == "lstm" else None
    h0 = (rng.standard_normal((B, H, 2) if cell == "lstm" else (B, H)) * 0.3).astype(np.float32)
    m = oracle.Model(cell, xp, a=a, peep=peep)
    for k in (1, 2, 3):
        out = solve.newton_forward(ctx.ctx, cell, B, T, H, xproj=gpu(xp), a=gpu(a),
                                   peep=None if peep is None else gpu(peep), h0=gpu(h0), max_iters=k, tol=0.0,
                                   residual=True)
        torch.cuda.synchronize()
        assert ctx.status() == 0
        assert int(out["iters"].item()) == k
        h_ref, _, _ = m.newton(h0, max_iters=k, tol=0.0)
        scale = max(1.0, float(np.abs(h_ref).max()))
        assert max_abs(host(out["h"]), h_ref) <= TOL_STATE * scale, k
        assert abs(float(out["residual"].item()) - m.residual(host(out["h"]), h0)) <= 1e-5 * scale


@pytest.mark.parametrize("cell,B,T,H", [("gru", 2, 700, 64), ("lstm", 3, 333, 64)])
def test_wide_converged_with_separate_residual(ctx, cell, B, T, H):
    """Wide layers (H % 32 == 0, xproj given) solved to tolerance: the solve stops before
    the cap, so the residual takes its own pass; several sequences and a ragged last
    tile (the staged box of the last tile reaches into the next sequence's rows)."""
    rng = np.random.default_rng(B * 11 + T + H)
    xp = (rng.standard_normal((B, T, 3, H)) * 0.8).astype(np.float32)
    a = rng.uniform(-0.9, 0.9, (3, H)).astype(np.float32)
    peep = rng.uniform(-0.5, 0.5, (2, H)).astype(np.float32) if cell == "lstm" else None
    h0 = (rng.standard_normal((B, H, 2) if cell == "lstm" else (B, H)) * 0.3).astype(np.float32)
    m = oracle.Model(cell, xp, a=a, peep=peep)
    h_ref, it_ref, _ = m.newton(h0, max_iters=T, tol=1e-6)
    out = solve.newton_forward(ctx.ctx, cell, B, T, H, xproj=gpu(xp), a=gpu(a),
                               peep=None if peep is None else gpu(peep), h0=gpu(h0), max_iters=T, tol=1e-6,
                               residual=True)
    torch.cuda.synchronize()
    assert ctx.status() == 0
    assert int(out["iters"].item()) == it_ref
    assert max_abs(host(out["h"]), h_ref) <= TOL_STATE
    assert abs(float(out["residual"].item()) - m.residual(host(out["h"]), h0)) <= 2e-6


@pytest.mark.parametrize("channels", [8, 16, 32])
@pytest.mark.parametrize("cell,B,T,H,iters,tol", [("gru", 4, 8000, 64, 3, 0.0), ("lstm", 3, 7001, 64, 7001, 1e-6),
                                                 ("gru", 2, 1000, 96, 2, 0.0)])
def test_wide_tile_widths(ctx, channels, cell, B, T, H, iters, tol):
    """Each channel width of the wide-layer tiles (8, 16, 32, forced through debug knob 6),
    capped with the fused residual (GRU) and converged (LSTM), ragged last tiles.  The
    first two shapes give every CTA more tiles than its staging ring holds (each stage is
    refilled), the last one at most two."""
    rng = np.random.default_rng(B * 13 + T + H)
    xp = (rng.standard_normal((B, T, 3, H)) * 0.8).astype(np.float32)
    a = rng.uniform(-0.9, 0.9, (3, H)).astype(np.float32)
    peep = rng.uniform(-0.5, 0.5, (2, H)).astype(np.float32) if cell == "lstm" else None
    h0 = (rng.standard_normal((B, H, 2) if cell == "lstm" else (B, H)) * 0.3).astype(np.float32)
    m = oracle.Model(cell, xp, a=a, peep=peep)
    h_ref, it_ref, _ = m.newton(h0, max_iters=iters, tol=tol)
    pararnn_debug_set(ctx.ctx, 6, channels)
    try:
        out = solve.newton_forward(ctx.ctx, cell, B, T, H, xproj=gpu(xp), a=gpu(a),
                                   peep=None if peep is None else gpu(peep), h0=gpu(h0), max_iters=iters, tol=tol,
                                   residual=True)
        torch.cuda.synchronize()
    finally:
        pararnn_debug_set(ctx.ctx, 6, 0)
    assert ctx.status() == 0
    assert int(out["iters"].item()) == it_ref
    scale = max(1.0, float(np.abs(h_ref).max()))
    assert max_abs(host(out["h"]), h_ref) <= TOL_STATE * scale
    assert abs(float(out["residual"].item()) - m.residual(host(out["h"]), h0)) <= 2e-6 * scale


def test_zero_iterations_returns_initial_guess(ctx):
    w = _small_workload("gru", 2, 100, 4, 2, 3)
    inp = wl.generate(w)
    out = _run_fused(ctx, w, inp, max_iters=0)
    assert int(out["iters"].item()) == 0
    assert float(out["h"].abs().max().item()) == 0.0


def test_cap_reached_reports_not_converged(ctx):
    w = wl.WORKLOADS["gru_b1_t1024_in4_h8"]
    inp = wl.generate(w)
    out = _run_fused(ctx, w, inp, max_iters=2)
    assert int(out["iters"].item()) == 2
    assert ctx.status() == PARARNN_NOTCONVERGED
    assert ctx.status() == 0  # cleared by the read


def test_repeated_calls_reuse_workspace(ctx):
    """Back-to-back calls of different shapes on one context give identical results."""
    w1 = _small_workload("gru", 3, 2000, 5, 2, 21)
    w2 = _small_workload("lstm", 2, 500, 33, 4, 22)
    i1, i2 = wl.generate(w1), wl.generate(w2)
    a = host(_run_fused(ctx, w1, i1)["h"])
    host(_run_fused(ctx, w2, i2)["h"])
    b = host(_run_fused(ctx, w1, i1)["h"])
    assert np.array_equal(a, b)
