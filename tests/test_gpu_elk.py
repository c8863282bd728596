"""GPU parity: ELK (Levenberg-Marquardt damped Newton by parallel Kalman filtering and
smoothing) for ParaGRU, the ParaLSTM with its full 2x2 Jacobian blocks (ELK) or their
diagonals (quasi-ELK, the lstm_quasi cell id), and the tanh RNN's Jacobian diagonal
(quasi-ELK).

GRU and LSTM run two passes per iteration (the filter as one associative scan of mean and
covariance, then the smoother backward); the tanh RNN three scans.  Bars: with tol = 0
and k iterations, the iterate within 1e-4 x max(1, |h|_max) of the oracle's (Kalman
filter + RTS smoother in fp64, pinned to a dense Levenberg-Marquardt solve); with a
tolerance, the oracle's iteration count and the converged states within 1e-4.  Shapes:
single channels over many tiles (look-back across 32 chunks), unit counts below and above
the 32-unit tile, raw inputs and projected inputs, tanh state sizes 5, 8 and 64; two
damping values.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import gpu, host, max_abs, need_gpu

from nonlinear_rnn_solve_b200 import Context, PararnnError, solve
from nonlinear_rnn_solve_b200 import workloads as wl

pytestmark = pytest.mark.gpu
TOL = 1e-4


@pytest.fixture(scope="module")
def ctx():
    need_gpu()
    c = Context(0)
    yield c
    c.close()


def _workload(cell, B, T, H, inp, seed):
    base = {"gru": "gru_b1_t1024_in4_h8", "lstm": "lstm_b4_t8192_h1024_bf16", "lstm_quasi": "lstm_b4_t8192_h1024_bf16",
            "tanh": "tanh_b16_t65536_in4_n8_deer"}[cell]
    return wl.WORKLOADS[base].resized(B=B, T=T, H=H, inp=inp, seed=seed, bf16=False, tol=1e-5,
                                      max_iters=T + 1, w_dist="uniform_fan_in")


def _run(ctx, cell, w, inp, lam, max_iters, tol, m=None, use_xproj=False):
    t = {k: gpu(v) for k, v in inp.items() if v is not None}
    kw = dict(a=t.get("a"), peep=t.get("peep"), A=t.get("A"), h0=t["h0"], max_iters=max_iters, tol=tol,
              solver="elk", damping=lam)
    if use_xproj:
        out = solve.newton_forward(ctx.ctx, cell, w.B, w.T, w.H, xproj=gpu(m.xproj.astype(np.float32)), **kw)
    else:
        out = solve.newton_forward(ctx.ctx, cell, w.B, w.T, w.H, x=t["x"], W=t["W"], bias=t["bias"], **kw)
    torch.cuda.synchronize()
    assert ctx.status() == 0
    return out


def _oracle(cell, inp, lam):
    """The oracle's ELK: lstm_quasi is the LSTM with each block's diagonal."""
    return oracle.model_from_inputs("lstm" if cell == "lstm_quasi" else cell, inp, quasi=cell == "lstm_quasi",
                                    solver="elk", damping=lam)


CASES = [  # (cell, B, T, H, in, xproj)
    ("gru", 2, 300, 5, 3, False),
    ("gru", 4, 65536, 1, 2, False),
    ("gru", 2, 500, 64, 4, True),
    ("lstm", 2, 300, 33, 4, False),
    ("lstm", 2, 400, 64, 4, True),
    ("lstm", 3, 5000, 1, 2, False),
    ("lstm_quasi", 2, 300, 33, 4, False),
    ("lstm_quasi", 2, 400, 64, 4, True),
    ("tanh", 3, 700, 8, 4, False),
    ("tanh", 2, 4096 + 33, 5, 4, False),
    ("tanh", 2, 300, 64, 4, True),
]


@pytest.mark.parametrize("lam", [0.5, 3.0])
@pytest.mark.parametrize("case", CASES)
def test_elk_iterates_match_oracle(ctx, lam, case):
    cell, B, T, H, inp_w, use_xproj = case
    w = _workload(cell, B, T, H, inp_w, seed=B * 13 + T + H)
    inp = wl.generate(w)
    m = _oracle(cell, inp, lam)
    for k in (1, 2, 5):
        out = _run(ctx, cell, w, inp, lam, k, 0.0, m, use_xproj)
        assert int(out["iters"].item()) == k
        h_ref, _, _ = m.newton(inp["h0"], max_iters=k, tol=0.0)
        scale = max(1.0, float(np.abs(h_ref).max()))
        assert max_abs(host(out["h"]), h_ref) <= TOL * scale, (lam, k)


@pytest.mark.parametrize("cell", ["gru", "lstm", "lstm_quasi", "tanh"])
def test_elk_converges_with_oracle_iteration_count(ctx, cell):
    w = _workload(cell, 2, 700, 8, 3, seed=3)
    inp = wl.generate(w)
    m = _oracle(cell, inp, 1.0)
    h_ref, it_ref, d_ref = m.newton(inp["h0"], max_iters=w.max_iters, tol=w.tol)
    out = _run(ctx, cell, w, inp, 1.0, w.max_iters, w.tol)
    assert int(out["iters"].item()) == it_ref, (int(out["iters"].item()), it_ref, d_ref)
    assert max_abs(host(out["h"]), h_ref) <= TOL


def test_elk_rejects_negative_damping_and_wide_dense_cells(ctx):
    w = _workload("gru", 1, 32, 2, 2, seed=1)
    inp = wl.generate(w)
    with pytest.raises(PararnnError):
        _run(ctx, "gru", w, inp, -1.0, 3, 0.0)
    tw = wl.WORKLOADS["tanh_b16_t65536_in4_n64_quasi"].resized(B=1, T=32, H=65)
    ti = {k: gpu(v) for k, v in wl.generate(tw).items() if v is not None}
    with pytest.raises(PararnnError):
        solve.newton_forward(ctx.ctx, "tanh_quasi", 1, 32, tw.H, x=ti["x"], W=ti["W"], bias=ti["bias"], A=ti["A"],
                             h0=ti["h0"], max_iters=3, tol=0.0, solver="elk", damping=1.0)


def test_tanh_elk_residual_and_both_cell_ids(ctx):
    """Either tanh cell id runs quasi-ELK; the residual output is max |h_t - f(h_{t-1})|
    at the result, as the oracle computes it."""
    w = _workload("tanh", 2, 500, 8, 4, seed=12)
    inp = wl.generate(w)
    m = oracle.model_from_inputs("tanh", inp, solver="elk", damping=0.7)
    t = {k: gpu(v) for k, v in inp.items() if v is not None}
    outs = []
    for cell in ("tanh", "tanh_quasi"):
        o = solve.newton_forward(ctx.ctx, cell, w.B, w.T, w.H, x=t["x"], W=t["W"], bias=t["bias"], A=t["A"],
                                 h0=t["h0"], max_iters=4, tol=0.0, solver="elk", damping=0.7, residual=True)
        torch.cuda.synchronize()
        assert ctx.status() == 0
        outs.append(o)
    h_ref, _, _ = m.newton(inp["h0"], max_iters=4, tol=0.0)
    for o in outs:
        assert max_abs(host(o["h"]), h_ref) <= TOL * max(1.0, float(np.abs(h_ref).max()))
        res = float(o["residual"].item())
        # |residual difference| <= (1 + max_i sum_j |A_ij|) x the state difference
        assert abs(res - m.residual(h_ref, inp["h0"])) <= 3e-4


@pytest.mark.parametrize("cell", ["gru", "lstm"])
def test_elk_withheld_publication_times_out(ctx, cell):
    """A tile withholds its published values (knob 2): a successor's bounded look-back
    wait runs out, the status reads ETIMEOUT, and the context recovers."""
    from nonlinear_rnn_solve_b200 import PARARNN_ETIMEOUT, pararnn_debug_set
    w = _workload(cell, 1, 6000, 1, 2, seed=5)
    inp = wl.generate(w)
    t = {k: gpu(v) for k, v in inp.items() if v is not None}
    kw = dict(x=t["x"], W=t["W"], bias=t["bias"], a=t["a"], peep=t.get("peep"), h0=t["h0"], solver="elk",
              damping=0.5)
    pararnn_debug_set(ctx.ctx, 1, 50_000_000)
    pararnn_debug_set(ctx.ctx, 2, 1)
    try:
        solve.newton_forward(ctx.ctx, cell, w.B, w.T, w.H, max_iters=3, tol=0.0, **kw)
        torch.cuda.synchronize()
        assert ctx.status() == PARARNN_ETIMEOUT
    finally:
        pararnn_debug_set(ctx.ctx, 2, -1)
        pararnn_debug_set(ctx.ctx, 1, 1_000_000_000)
    out = _run(ctx, cell, w, inp, 0.5, 3, 0.0)
    h_ref, _, _ = _oracle(cell, inp, 0.5).newton(inp["h0"], max_iters=3, tol=0.0)
    assert max_abs(host(out["h"]), h_ref) <= TOL * max(1.0, float(np.abs(h_ref).max()))
