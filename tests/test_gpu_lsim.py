"""GPU parity: fixed-step linear simulation (lsim) against the fp64 oracle.

The device discretises the ODE in fp64 and runs the recurrence in fp32.  With the
contraction rate rho = |e^{A h}| < 1, each step's rounding (about (n + m) 2^-24 of the
state) is damped geometrically, so the accumulated error stays below
(n + m) 2^-24 max|x| / (1 - rho); the systems here have 1 - rho >= 0.03, which bounds
it by 1e-4 x max(1, max|y|), the bar used (an integrator, rho = 1, grows T 2^-24 and
stays inside it at T = 1025).  Shapes: T = 1 and T against the 32-step chunk (31, 33,
1025; 40000 = three chunk levels), state sizes padded 1 -> 32, the largest m and p,
both input holds, with and without x0, D and the state output.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import gpu, host, need_gpu

from nonlinear_rnn_solve_b200 import Context, PararnnError, solve

pytestmark = pytest.mark.gpu
TOL = 1e-4


@pytest.fixture(scope="module")
def ctx():
    need_gpu()
    c = Context(0)
    yield c
    c.close()


def _system(n, m, p, seed, shift=1.5):
    rng = np.random.default_rng(seed)
    A = (rng.standard_normal((n, n)) * 0.5 / np.sqrt(n) - shift * np.eye(n)).astype(np.float32)
    B = rng.standard_normal((n, m)).astype(np.float32)
    C = rng.standard_normal((p, n)).astype(np.float32)
    D = rng.standard_normal((p, m)).astype(np.float32)
    return A, B, C, D, rng


def _close(got, ref):
    scale = max(1.0, float(np.abs(ref).max()))
    return float(np.abs(host(got) - ref).max()) <= TOL * scale


CASES = [  # (batch, T, n, m, p, h)
    (1, 1, 1, 1, 1, 0.1),
    (2, 31, 3, 2, 2, 0.05),
    (3, 33, 8, 1, 5, 0.05),
    (2, 1025, 17, 4, 3, 0.03),
    (1, 40000, 2, 1, 1, 0.05),
    (2, 300, 32, 16, 32, 0.05),
    (4, 5000, 16, 4, 4, 0.05),
]


@pytest.mark.parametrize("interp", ["zoh", "foh"])
@pytest.mark.parametrize("case", CASES)
def test_lsim_matches_oracle(ctx, interp, case):
    batch, T, n, m, p, h = case
    A, B, C, D, rng = _system(n, m, p, seed=batch * 7 + T + n)
    U = rng.standard_normal((batch, T, m)).astype(np.float32)
    x0 = rng.standard_normal((batch, n)).astype(np.float32)
    t = np.arange(T) * h
    y, x = solve.lsim(ctx.ctx, gpu(A), gpu(B), gpu(C), gpu(D), gpu(U), t, x0=gpu(x0), interp=interp)
    torch.cuda.synchronize()
    yr, xr = oracle.lsim(A, B, C, D, U, h, x0=x0, interp=interp)
    assert _close(y, yr) and _close(x, xr)


def test_optional_inputs_and_outputs(ctx):
    """No x0 (rest), no D (no feedthrough), no state output, a single sequence."""
    A, B, C, _, rng = _system(5, 2, 3, seed=4)
    U = rng.standard_normal((777, 2)).astype(np.float32)
    t = np.arange(777) * 0.02
    y, x = solve.lsim(ctx.ctx, gpu(A), gpu(B), gpu(C), None, gpu(U), t, interp="foh", return_states=False)
    torch.cuda.synchronize()
    assert x is None and y.shape == (777, 3)
    yr, _ = oracle.lsim(A, B, C, None, U, 0.02, interp="foh")
    assert _close(y, yr)


def test_integrator_marginal_case(ctx):
    """A = 0: the states are running sums of the input (rho = 1, nothing is damped)."""
    n = 4
    rng = np.random.default_rng(8)
    U = rng.standard_normal((2, 1025, n)).astype(np.float32)
    A = np.zeros((n, n), np.float32)
    I = np.eye(n, dtype=np.float32)
    for interp in ("zoh", "foh"):
        y, _ = solve.lsim(ctx.ctx, gpu(A), gpu(I), gpu(I), None, gpu(U), np.arange(1025) * 0.1, interp=interp)
        torch.cuda.synchronize()
        yr, _ = oracle.lsim(A, I, I, None, U, 0.1, interp=interp)
        assert _close(y, yr)


def test_readme_example(ctx):
    """A = -0.5, B = C = 1, D = 0 on 128 points of [0, 1]: from x0 = 2 with zero input
    the output is 2 e^{-t/2}."""
    t = np.linspace(0.0, 1.0, 128)
    one = np.ones((1, 1), np.float32)
    y, _ = solve.lsim(ctx.ctx, gpu(-0.5 * one), gpu(one), gpu(one), gpu(0 * one), gpu(np.zeros((128, 1), np.float32)),
                      t, x0=gpu(np.array([2.0], np.float32)))
    torch.cuda.synchronize()
    assert float(np.abs(host(y)[:, 0] - 2.0 * np.exp(-0.5 * t)).max()) <= 1e-5


def test_full_size_sampled(ctx):
    """1024 sequences of 16384 steps, n = 16, m = p = 4 (the measured shape): four
    sampled sequences against the oracle."""
    batch, T, n, m, p, h = 1024, 16384, 16, 4, 4, 0.05
    A, B, C, D, _ = _system(n, m, p, seed=99)
    g = torch.Generator(device="cuda").manual_seed(3)
    U = torch.randn(batch, T, m, device="cuda", generator=g)
    y, _ = solve.lsim(ctx.ctx, gpu(A), gpu(B), gpu(C), gpu(D), U, np.arange(T) * h, interp="foh",
                      return_states=False)
    torch.cuda.synchronize()
    rows = [0, 1, 517, batch - 1]
    yr, _ = oracle.lsim(A, B, C, D, host(U[rows]), h, interp="foh")
    assert _close(y[rows], yr)


def test_rejects_unsupported_shapes(ctx):
    A, B, C, D, _ = _system(33, 1, 1, seed=1)
    U = gpu(np.zeros((1, 8, 1), np.float32))
    with pytest.raises(PararnnError):
        solve.lsim(ctx.ctx, gpu(A), gpu(B), gpu(C), gpu(D), U, np.arange(8) * 0.1)
    A, B, C, D, _ = _system(2, 1, 1, seed=1)
    with pytest.raises(PararnnError):  # dt = 0
        solve.lsim(ctx.ctx, gpu(A), gpu(B), gpu(C), gpu(D), U, np.zeros(8))
    with pytest.raises(ValueError):  # not a fixed-step grid
        solve.lsim(ctx.ctx, gpu(A), gpu(B), gpu(C), gpu(D), U, np.array([0, 1, 2, 3, 5, 6, 7, 8.0]))
