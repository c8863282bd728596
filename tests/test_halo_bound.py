"""Host check of the halo carry's premise on the benchmark inputs (no GPU).

A long tile takes its carry from its own evaluation of the steps before it when every
entry of their composed Jacobian is at most 2^-40 in magnitude; otherwise it waits for
the look-back, which is correct but slow.  These tests measure, with the fp64 oracle,
the largest such product over the windows the kernels use -- at the first iterate
(h = 0) and at the solution (the rollout) -- so that a change of inputs or halo length
that would send tiles back to the look-back shows up here:
  - ParaGRU, B16 T2^20 H1 in2: the 63 steps before each 4096-step tile;
  - tanh RNN quasi-DEER, B16 T65536 n8 in4: the 128 steps before each 512-step tile,
    per unit (the quasi-Jacobian (1 - f^2) A_ii).
The Jacobian formulas used here are first checked against the oracle's step Jacobian.
"""
import numpy as np
import pytest

import oracle
from nonlinear_rnn_solve_b200 import workloads as wl

LIMIT = -40.0  # log2 of the carry test's bound


def _windows(lj, starts, L):
    c = np.concatenate([np.zeros_like(lj[:, :1]), np.cumsum(lj, axis=1)], axis=1)
    return c[:, starts] - c[:, starts - L]


def _sig(u):
    return 1.0 / (1.0 + np.exp(-u))


@pytest.fixture(scope="module")
def gru():
    w = wl.WORKLOADS["gru_b16_t1048576_in2_h1"]
    inp = wl.generate(w)
    m = oracle.model_from_inputs("gru", inp)
    p = oracle.input_proj(inp["x"], inp["W"], inp.get("bias")).reshape(w.B, w.T, 3)
    a = np.asarray(inp["a"], dtype=np.float64).reshape(3)
    h0 = np.zeros((w.B, 1)) if inp.get("h0") is None else np.asarray(inp["h0"], np.float64).reshape(w.B, 1)
    h = m.rollout(inp.get("h0"))[..., 0]
    hprev = np.concatenate([h0, h[:, :-1]], axis=1)
    return w, m, p, a, hprev


def _gru_jac(p, a, hh):
    z = _sig(p[..., 0] + a[0] * hh)
    r = _sig(p[..., 1] + a[1] * hh)
    c = np.tanh(p[..., 2] + a[2] * r * hh)
    return (1 - z) + (c - hh) * z * (1 - z) * a[0] + z * (1 - c * c) * a[2] * (r + hh * r * (1 - r) * a[1])


def test_gru_jacobian_formula_matches_the_oracle(gru):
    w, m, p, a, hprev = gru
    rng = np.random.default_rng(0)
    for _ in range(8):
        b, t = int(rng.integers(w.B)), int(rng.integers(w.T))
        _, J = m.step(b, t, hprev[b, t:t + 1])
        assert abs(float(J[0, 0]) - float(_gru_jac(p[b, t], a, hprev[b, t]))) <= 1e-12


@pytest.mark.parametrize("at", ["first_iterate", "solution"])
def test_gru_63_step_halo_products_below_the_bound(gru, at):
    w, _, p, a, hprev = gru
    hh = np.zeros_like(hprev) if at == "first_iterate" else hprev
    lj = np.log2(np.abs(_gru_jac(p, a, hh)) + 1e-300)
    worst = float(_windows(lj, np.arange(4096, w.T, 4096), 63).max())
    assert worst < LIMIT, worst


@pytest.mark.parametrize("at", ["first_iterate", "solution"])
def test_tanh_n8_128_step_halo_products_below_the_bound(at):
    w = wl.WORKLOADS["tanh_b16_t65536_in4_n8_quasi"]
    inp = wl.generate(w)
    A = np.asarray(inp["A"], np.float64)
    p = oracle.input_proj(inp["x"], inp["W"], inp.get("bias"))  # [B, T, 8]
    h0 = np.zeros((w.B, 8)) if inp.get("h0") is None else np.asarray(inp["h0"], np.float64)
    if at == "first_iterate":
        hh = np.zeros((w.B, w.T, 8))
    else:
        m = oracle.model_from_inputs("tanh", inp, quasi=True)
        h = m.rollout(inp.get("h0"))
        hh = np.concatenate([h0[:, None], h[:, :-1]], axis=1)
    f = np.tanh(hh @ A.T + p)
    lj = np.log2(np.abs((1 - f * f) * np.diag(A)) + 1e-300)
    worst = float(_windows(lj, np.arange(512, w.T, 512), 128).max())
    assert worst < LIMIT, worst
