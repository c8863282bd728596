"""GPU parity: the Jacobi (J = 0) and Picard (J = I) fixed-point schemes.

They run in the Newton kernels with the linearisation replaced, so every layout is
exercised: the generic kernel, the TMA-fed H = 1 ParaGRU tiles (whose halo is then
constant for Jacobi and never for Picard, which takes the look-back path), the
32-unit staged layout, and the tanh RNN's diagonal kernel.  Bars: with tol = 0 and k
iterations, the iterate within 1e-4 x max(1, |h|_max) of the oracle's (Picard: within
max(1e-4, 4 T 2^-24) x max(1, |h|_max), the fp32 bound of a running sum over T steps,
since J = I carries every rounding error to the end of the sequence); with a
tolerance on short sequences, the oracle's iteration count and the rollout within
1e-4.  Picard iterates grow like sums over the unconverged suffix (the tanh RNN's
reach 1e9 at T = 40), so its convergence case is T = 12, where fp32 still resolves
the tolerance; Jacobi's uses T = 40.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import gpu, host, max_abs, need_gpu

from nonlinear_rnn_solve_b200 import Context, solve
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
    base = {"gru": "gru_b1_t1024_in4_h8", "lstm": "lstm_b4_t8192_h1024_bf16",
            "tanh": "tanh_b16_t65536_in4_n8_deer"}[cell]
    return wl.WORKLOADS[base].resized(B=B, T=T, H=H, inp=inp, seed=seed, bf16=False, tol=1e-5,
                                      max_iters=T + 1, w_dist="uniform_fan_in")


def _run(ctx, cell, w, inp, solver, max_iters, tol, use_xproj=False, m=None):
    t = {k: gpu(v) for k, v in inp.items() if v is not None}
    kw = dict(a=t.get("a"), peep=t.get("peep"), A=t.get("A"), h0=t["h0"], max_iters=max_iters, tol=tol,
              solver=solver)
    if use_xproj:
        xp = gpu(m.xproj.astype(np.float32))
        out = solve.newton_forward(ctx.ctx, cell, w.B, w.T, w.H, xproj=xp, **kw)
    else:
        out = solve.newton_forward(ctx.ctx, cell, w.B, w.T, w.H, x=t["x"], W=t["W"], bias=t["bias"], **kw)
    torch.cuda.synchronize()
    assert ctx.status() == 0
    return out


CASES = [  # (cell, B, T, H, in, xproj)
    ("gru", 2, 300, 5, 3, False),
    ("gru", 2, 2 * 4096 + 32, 1, 2, False),
    ("gru", 2, 500, 64, 4, True),
    ("lstm", 2, 300, 33, 4, False),
    ("lstm", 1, 4096, 1, 2, False),
    ("lstm", 2, 400, 64, 4, True),
    ("tanh", 3, 700, 8, 4, False),
    ("tanh", 2, 600, 48, 4, False),   # 32 < n <= 64: the tensor-core cell product
    ("tanh", 2, 300, 64, 4, True),
]


@pytest.mark.parametrize("solver", ["jacobi", "picard"])
@pytest.mark.parametrize("case", CASES)
def test_fixed_iterations_match_oracle(ctx, solver, case):
    cell, B, T, H, inp_w, use_xproj = case
    w = _workload(cell, B, T, H, inp_w, seed=B * 31 + T + H)
    inp = wl.generate(w)
    m = oracle.model_from_inputs(cell, inp, solver=solver)
    for k in (1, 3, 7):
        out = _run(ctx, cell, w, inp, solver, k, 0.0, use_xproj, m)
        assert int(out["iters"].item()) == k
        h_ref, _, _ = m.newton(inp["h0"], max_iters=k, tol=0.0)
        scale = max(1.0, float(np.abs(h_ref).max()))
        rel = TOL if solver == "jacobi" else max(TOL, 4 * T * 2.0 ** -24)
        assert max_abs(host(out["h"]), h_ref) <= rel * scale, (solver, k)


@pytest.mark.parametrize("solver", ["jacobi", "picard"])
@pytest.mark.parametrize("cell", ["gru", "lstm", "tanh"])
def test_converges_to_rollout_with_oracle_iteration_count(ctx, solver, cell):
    w = _workload(cell, 2, 40 if solver == "jacobi" else 12, 4, 3, seed=7)
    inp = wl.generate(w)
    m = oracle.model_from_inputs(cell, inp, solver=solver)
    h_ref, it_ref, _ = m.newton(inp["h0"], max_iters=w.max_iters, tol=w.tol)
    out = _run(ctx, cell, w, inp, solver, w.max_iters, w.tol)
    assert int(out["iters"].item()) == it_ref
    assert max_abs(host(out["h"]), m.rollout(inp["h0"])) <= TOL
