"""Pins for the oracle's fixed-step linear simulation (lsim): closed forms, exact sums,
an independent RK4 integration of the continuous system, and scipy's own lsim.

The oracle discretises dx/dt = A x + B u over one step with a matrix exponential and
steps the recurrence in fp64; these checks reach the same numbers by other routes, so
a dropped input term, a swapped hold weight, a transposed A or C, or a missing D fails
one of them.
"""
import numpy as np
import pytest
import scipy.signal

import oracle


def _grid(T, h):
    return np.arange(T) * h


@pytest.mark.parametrize("a,b,c,d", [(-0.5, 1.0, 1.0, 0.0), (-2.0, 0.7, -1.3, 0.4), (0.3, -1.1, 2.0, -0.2)])
def test_scalar_held_input_matches_closed_form(a, b, c, d):
    """x' = a x + b u with u constant: x(t) = e^{at} x0 + (b u / a)(e^{at} - 1)."""
    T, h, u, x0 = 200, 0.013, 0.8, 1.7
    t = _grid(T, h)
    y, x = oracle.lsim([[a]], [[b]], [[c]], [[d]], np.full((T, 1), u), h, x0=[x0], interp="zoh")
    xe = np.exp(a * t) * x0 + (b * u / a) * (np.exp(a * t) - 1.0)
    assert np.abs(x[:, 0] - xe).max() < 1e-12
    assert np.abs(y[:, 0] - (c * xe + d * u)).max() < 1e-12


@pytest.mark.parametrize("a,b", [(-0.5, 1.0), (-3.0, 2.0), (0.4, -0.6)])
def test_scalar_ramp_input_is_exact_with_linear_hold(a, b):
    """x' = a x + b t: x(t) = e^{at}(x0 + b/a^2) - b t / a - b / a^2; the linear hold
    is exact for a ramp, the constant hold is not."""
    T, h, x0 = 150, 0.02, -0.4
    t = _grid(T, h)
    xe = np.exp(a * t) * (x0 + b / a**2) - b * t / a - b / a**2
    _, x = oracle.lsim([[a]], [[b]], [[1.0]], None, t[:, None], h, x0=[x0], interp="foh")
    assert np.abs(x[:, 0] - xe).max() < 1e-12
    _, xz = oracle.lsim([[a]], [[b]], [[1.0]], None, t[:, None], h, x0=[x0], interp="zoh")
    assert np.abs(xz[:, 0] - xe).max() > 1e-5


def test_integrator_gives_riemann_and_trapezoid_sums():
    """A = 0, B = I: the held input integrates to the left Riemann sum, the linear
    one to the trapezoid rule."""
    rng = np.random.default_rng(0)
    T, h, n = 64, 0.1, 2
    U = rng.standard_normal((T, n))
    x0 = np.array([0.5, -1.0])
    _, xz = oracle.lsim(np.zeros((n, n)), np.eye(n), np.eye(n), None, U, h, x0=x0, interp="zoh")
    left = x0 + h * np.vstack([np.zeros(n), np.cumsum(U[:-1], axis=0)])
    assert np.abs(xz - left).max() < 1e-12
    _, xf = oracle.lsim(np.zeros((n, n)), np.eye(n), np.eye(n), None, U, h, x0=x0, interp="foh")
    trap = x0 + np.vstack([np.zeros(n), np.cumsum(0.5 * h * (U[:-1] + U[1:]), axis=0)])
    assert np.abs(xf - trap).max() < 1e-12


def _rk4(A, B, C, D, U, h, x0, interp, sub=200):
    """Classical RK4 on the continuous system with `sub` substeps per sample interval;
    the input between samples is held (zoh) or interpolated linearly (foh)."""
    T = U.shape[0]
    x = np.array(x0, dtype=np.float64)
    xs = [x.copy()]
    dt = h / sub
    for k in range(T - 1):
        u0, u1 = U[k], U[k + 1]
        uf = (lambda s: u0) if interp == "zoh" else (lambda s: u0 + (s / h) * (u1 - u0))
        f = lambda s, x: A @ x + B @ uf(s)
        for j in range(sub):
            s = j * dt
            k1 = f(s, x)
            k2 = f(s + dt / 2, x + dt / 2 * k1)
            k3 = f(s + dt / 2, x + dt / 2 * k2)
            k4 = f(s + dt, x + dt * k3)
            x = x + dt / 6 * (k1 + 2 * k2 + 2 * k3 + k4)
        xs.append(x.copy())
    xs = np.array(xs)
    return xs @ C.T + U @ D.T, xs


@pytest.mark.parametrize("interp", ["zoh", "foh"])
def test_general_system_matches_rk4(interp):
    """n = 3, m = 2, p = 2 with a non-symmetric A and non-square C, D."""
    rng = np.random.default_rng(5)
    n, m, p, T, h = 3, 2, 2, 40, 0.05
    A = rng.standard_normal((n, n)) - 1.0 * np.eye(n)
    B = rng.standard_normal((n, m))
    C = rng.standard_normal((p, n))
    D = rng.standard_normal((p, m))
    U = rng.standard_normal((T, m))
    x0 = rng.standard_normal(n)
    y, x = oracle.lsim(A, B, C, D, U, h, x0=x0, interp=interp)
    yr, xr = _rk4(A, B, C, D, U, h, x0, interp)
    assert np.abs(x - xr).max() < 1e-9
    assert np.abs(y - yr).max() < 1e-9


@pytest.mark.parametrize("interp", ["zoh", "foh"])
def test_agrees_with_scipy_lsim(interp):
    rng = np.random.default_rng(9)
    n, m, p, T, h = 4, 3, 2, 120, 0.03
    A = rng.standard_normal((n, n)) / 2 - 0.8 * np.eye(n)
    B, C, D = rng.standard_normal((n, m)), rng.standard_normal((p, n)), rng.standard_normal((p, m))
    U = rng.standard_normal((T, m))
    x0 = rng.standard_normal(n)
    t = _grid(T, h)
    _, ys, xs = scipy.signal.lsim((A, B, C, D), U, t, X0=x0, interp=(interp == "foh"))
    y, x = oracle.lsim(A, B, C, D, U, h, x0=x0, interp=interp)
    assert np.abs(x - xs).max() < 1e-9 and np.abs(y - ys).max() < 1e-9


def test_readme_example_decays_like_the_exponential():
    """The README's system (A = -0.5, B = C = 1, D = 0, 128 points on [0, 1], zero
    input): y = 0 from rest, and y = e^{-t/2} x0 from x0."""
    t = np.linspace(0.0, 1.0, 128)
    h = t[1] - t[0]
    y, _ = oracle.lsim([[-0.5]], [[1.0]], [[1.0]], [[0.0]], np.zeros((128, 1)), h)
    assert np.abs(y).max() == 0.0
    y, _ = oracle.lsim([[-0.5]], [[1.0]], [[1.0]], [[0.0]], np.zeros((128, 1)), h, x0=[2.0])
    assert np.abs(y[:, 0] - 2.0 * np.exp(-0.5 * t)).max() < 1e-13


def test_batch_rows_are_independent_runs():
    rng = np.random.default_rng(2)
    n, m, p, T, h = 2, 1, 3, 30, 0.1
    A = rng.standard_normal((n, n)) - np.eye(n)
    B, C = rng.standard_normal((n, m)), rng.standard_normal((p, n))
    U = rng.standard_normal((3, T, m))
    x0 = rng.standard_normal((3, n))
    y, x = oracle.lsim(A, B, C, None, U, h, x0=x0, interp="foh")
    for i in range(3):
        yi, xi = oracle.lsim(A, B, C, np.zeros((p, m)), U[i], h, x0=x0[i], interp="foh")
        assert np.array_equal(y[i], yi) and np.array_equal(x[i], xi)


@pytest.mark.parametrize("interp", ["zoh", "foh"])
def test_chunk_end_state_is_a_fixed_linear_map_of_its_inputs(interp):
    """From a zero state before step k0, the state after 32 steps is
    sum_{l=-1}^{31} K_l u_{k0+l} with K_l = Ad^(30-l) (G0 + Ad G1) for 0 <= l <= 30,
    K_31 = G1 and K_{-1} = Ad^31 G0: the identity the first scan pass contracts with."""
    rng = np.random.default_rng(17)
    n, m, h = 4, 3, 0.07
    A = rng.standard_normal((n, n)) * 0.4 - np.eye(n)
    B = rng.standard_normal((n, m))
    Ad, G0, G1 = oracle.lsim_discretize(A, B, h, interp)
    u = rng.standard_normal((33, m))  # u_{k0-1} .. u_{k0+31}
    x = np.zeros(n)
    for i in range(32):  # steps k0 .. k0 + 31, each from u_{k-1} and u_k
        x = Ad @ x + G0 @ u[i] + G1 @ u[i + 1]
    P = np.linalg.matrix_power
    K = {l: P(Ad, 30 - l) @ (G0 + Ad @ G1) for l in range(31)}
    K[31], K[-1] = G1, P(Ad, 31) @ G0
    y = sum(K[l] @ u[l + 1] for l in range(-1, 32))
    assert np.abs(x - y).max() < 1e-12
