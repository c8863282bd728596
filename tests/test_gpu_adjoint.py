"""GPU parity: adjoint backward (reverse scan + gradients) against the fp64 oracle.

grad_xproj and grad_h0 within 1e-4 relative to their max magnitude; the recurrent
parameter gradients (sums over B*T terms, float atomics) within 1e-4 relative.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import gpu, host, need_gpu

from nonlinear_rnn_solve_b200 import Context, solve

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ctx():
    need_gpu()
    c = Context(0)
    yield c
    c.close()


def _rel(a, b):
    return float(np.max(np.abs(a - b)) / max(1.0, np.max(np.abs(b))))


@pytest.mark.parametrize("cell,B,T,H", [("gru", 2, 777, 40), ("gru", 3, 2000, 1), ("gru", 1, 1, 1),
                                        ("gru", 2, 300, 8), ("lstm", 2, 500, 33), ("lstm", 1, 1200, 1),
                                        ("lstm", 2, 257, 64)])
def test_adjoint_matches_oracle(ctx, cell, B, T, H):
    rng = np.random.default_rng(T * 13 + H)
    xp = (rng.standard_normal((B, T, 3, H)) * 0.8).astype(np.float32)
    a = rng.uniform(-0.9, 0.9, (3, H)).astype(np.float32)
    peep = rng.uniform(-0.5, 0.5, (2, H)).astype(np.float32) if cell == "lstm" else None
    sshape = (B, T, H, 2) if cell == "lstm" else (B, T, H)
    h0 = (rng.standard_normal(sshape[:1] + sshape[2:]) * 0.3).astype(np.float32)
    h = np.tanh(rng.standard_normal(sshape)).astype(np.float32)   # any states
    g = rng.standard_normal(sshape).astype(np.float32)
    gx, gp, gh0 = solve.adjoint_backward(ctx.ctx, cell, B, T, H, xproj=gpu(xp), a=gpu(a),
                                         peep=None if peep is None else gpu(peep), h0=gpu(h0), h=gpu(h),
                                         grad_h=gpu(g))
    torch.cuda.synchronize()
    assert ctx.status() == 0
    m = oracle.Model(cell, xp, a=a, peep=peep)
    rx, rp, rh0 = m.adjoint(h, g, h0)
    assert _rel(host(gx), rx) <= 1e-4
    assert _rel(host(gp), rp) <= 1e-4
    assert _rel(host(gh0), rh0) <= 1e-4


def test_adjoint_at_newton_solution(ctx):
    """Forward solve then adjoint on the solver's own states (the training path)."""
    B, T, H = 2, 3000, 16
    rng = np.random.default_rng(5)
    xp = (rng.standard_normal((B, T, 3, H))).astype(np.float32)
    a = rng.uniform(-0.5, 0.5, (3, H)).astype(np.float32)
    g = rng.standard_normal((B, T, H)).astype(np.float32)
    out = solve.newton_forward(ctx.ctx, "gru", B, T, H, xproj=gpu(xp), a=gpu(a), max_iters=T, tol=1e-6)
    gx, gp, gh0 = solve.adjoint_backward(ctx.ctx, "gru", B, T, H, xproj=gpu(xp), a=gpu(a), h=out["h"],
                                         grad_h=gpu(g))
    torch.cuda.synchronize()
    assert ctx.status() == 0
    m = oracle.Model("gru", xp, a=a)
    h_ref = m.rollout()
    rx, rp, rh0 = m.adjoint(h_ref, g)
    assert _rel(host(gx), rx) <= 1e-4
    assert _rel(host(gp), rp) <= 1e-4
