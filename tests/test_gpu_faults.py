"""Device-side failure detection without faulting the GPU.

* A look-back publication withheld by the test knob makes the successor's bounded
  wait run out (limit 50 ms); the kernel returns, the status reads ETIMEOUT and
  the context keeps working.
* A NaN in the inputs is reported as ENONFINITE after the iteration that met it.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import gpu, host, max_abs, need_gpu

from nonlinear_rnn_solve_b200 import (PARARNN_ENONFINITE, PARARNN_ETIMEOUT, Context, pararnn_debug_set,
                                      solve)

pytestmark = pytest.mark.gpu


@pytest.fixture()
def ctx():
    need_gpu()
    c = Context(0)
    yield c
    c.close()


def test_withheld_publication_times_out_and_context_recovers(ctx):
    B, T, N = 1, 3 * 4096, 1  # three tiles of one sequence; tile 0 never publishes
    rng = np.random.default_rng(1)
    J = rng.uniform(-1, 1, (B, T, N)).astype(np.float32)
    b = rng.standard_normal((B, T, N)).astype(np.float32)
    pararnn_debug_set(ctx.ctx, 1, 50_000_000)
    pararnn_debug_set(ctx.ctx, 2, 0)
    solve.linear_scan(ctx.ctx, "diag", gpu(J), gpu(b))
    torch.cuda.synchronize()
    assert ctx.status() == PARARNN_ETIMEOUT
    pararnn_debug_set(ctx.ctx, 2, -1)
    out = solve.linear_scan(ctx.ctx, "diag", gpu(J), gpu(b))
    torch.cuda.synchronize()
    assert ctx.status() == 0
    assert max_abs(host(out), oracle.linear_scan("diag", J, b)) <= 1e-5


def test_withheld_publication_in_newton_times_out(ctx):
    B, T, H = 2, 3 * 4096, 1
    rng = np.random.default_rng(2)
    xp = rng.standard_normal((B, T, 3, H)).astype(np.float32)
    a = rng.uniform(-0.5, 0.5, (3, H)).astype(np.float32)
    pararnn_debug_set(ctx.ctx, 1, 50_000_000)
    pararnn_debug_set(ctx.ctx, 2, 1)
    solve.newton_forward(ctx.ctx, "gru", B, T, H, xproj=gpu(xp), a=gpu(a), max_iters=10, tol=1e-6)
    torch.cuda.synchronize()
    assert ctx.status() == PARARNN_ETIMEOUT
    pararnn_debug_set(ctx.ctx, 2, -1)
    out = solve.newton_forward(ctx.ctx, "gru", B, T, H, xproj=gpu(xp), a=gpu(a), max_iters=T, tol=1e-6)
    torch.cuda.synchronize()
    assert ctx.status() == 0
    h_ref, it_ref, _ = oracle.Model("gru", xp, a=a).newton(max_iters=T, tol=1e-6)
    assert int(out["iters"].item()) == it_ref
    assert max_abs(host(out["h"]), h_ref) <= 1e-4


def test_withheld_publication_in_wide_newton_times_out(ctx):
    """The wide-layer kernel (H % 32 == 0, xproj given): tile 1 of 3 withholds its
    publication, tile 2's bounded wait runs out, and the context recovers."""
    B, T, H = 1, 3 * 128, 32
    rng = np.random.default_rng(4)
    xp = rng.standard_normal((B, T, 3, H)).astype(np.float32)
    a = rng.uniform(-0.5, 0.5, (3, H)).astype(np.float32)
    pararnn_debug_set(ctx.ctx, 1, 50_000_000)
    pararnn_debug_set(ctx.ctx, 2, 1)
    solve.newton_forward(ctx.ctx, "gru", B, T, H, xproj=gpu(xp), a=gpu(a), max_iters=10, tol=1e-6)
    torch.cuda.synchronize()
    assert ctx.status() == PARARNN_ETIMEOUT
    pararnn_debug_set(ctx.ctx, 2, -1)
    out = solve.newton_forward(ctx.ctx, "gru", B, T, H, xproj=gpu(xp), a=gpu(a), max_iters=T, tol=1e-6)
    torch.cuda.synchronize()
    assert ctx.status() == 0
    h_ref, it_ref, _ = oracle.Model("gru", xp, a=a).newton(max_iters=T, tol=1e-6)
    assert int(out["iters"].item()) == it_ref
    assert max_abs(host(out["h"]), h_ref) <= 1e-4


@pytest.mark.parametrize("H", [4, 64])
def test_nan_input_reports_nonfinite(ctx, H):
    B, T = 1, 500
    rng = np.random.default_rng(3)
    xp = rng.standard_normal((B, T, 3, H)).astype(np.float32)
    xp[0, 123, 1, 2] = np.nan
    a = rng.uniform(-0.5, 0.5, (3, H)).astype(np.float32)
    out = solve.newton_forward(ctx.ctx, "gru", B, T, H, xproj=gpu(xp), a=gpu(a), max_iters=50, tol=1e-6)
    torch.cuda.synchronize()
    assert ctx.status() == PARARNN_ENONFINITE
    assert int(out["iters"].item()) == 1
