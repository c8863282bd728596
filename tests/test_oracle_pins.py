"""Pins of the fp64 oracle against things other than itself (CPU only).

Each check is chosen so that a plausible slip in the oracle (a dropped term, a
wrong sign or index, a transposed operand) fails at least one of them:
  * cells and rollouts  == PyTorch's reference GRU / LSTM / RNN cells, wired to the
    diagonal ParaGRU, CIFG + peephole ParaLSTM and vanilla tanh RNN;
  * Jacobians           == autograd Jacobians of those library cells;
  * linear recurrences  == dense solves of the block-bidiagonal system, and the
    closed form of a constant scalar recurrence;
  * Newton iterates     == Newton on the stacked residual system with a dense
    solve (DEER: "Parallelizing non-linear sequential models over the sequence
    length", Approach; ParaRNN abstract: one system of equations, Newton);
    quasi-Newton keeps only the diagonal of each Jacobian block ("Towards
    Scalable and Stable Parallelization of Nonlinear RNNs", Abstract);
  * invariants: after k updates the first k states are exact; the fixed point is
    the rollout; an affine cell converges in one update; quadratic convergence;
  * adjoint             == autograd through the library rollout (converged) and the
    implicit-function gradient from a dense transposed solve (any states).
"""
import numpy as np
import pytest
import torch

import oracle
import torch_cells as tc
from nonlinear_rnn_solve_b200 import workloads as wl

f64 = torch.float64


def _rand_model(cell, B, T, H, seed, scale=1.0, quasi=False, peep=True):
    rng = np.random.default_rng(seed)
    G = 1 if cell == "tanh" else 3
    xp = rng.standard_normal((B, T, G, H)) * scale
    prm = {}
    if cell != "tanh":
        prm["a"] = rng.uniform(-0.9, 0.9, size=(3, H))
    if cell == "lstm":
        prm["peep"] = rng.uniform(-0.8, 0.8, size=(2, H)) if peep else np.zeros((2, H))
    if cell == "tanh":
        prm["A"] = rng.standard_normal((H, H)) * (0.9 / np.sqrt(H))
    m = oracle.Model(cell, xp, quasi=quasi, **prm)
    h0 = rng.standard_normal(m.h0_shape) * 0.5
    return m, xp, prm, h0


CELLS = ["gru", "lstm", "tanh"]


def _lib(cell, H, prm):
    return tc.make(cell, H, prm)


# ---------------------------------------------------------------------------- cells
@pytest.mark.parametrize("cell", CELLS)
def test_rollout_matches_library_cell(cell):
    m, xp, prm, h0 = _rand_model(cell, B=3, T=40, H=5, seed=1)
    ref = tc.rollout(_lib(cell, 5, prm), torch.tensor(xp), torch.tensor(h0)).numpy()
    np.testing.assert_allclose(m.rollout(h0), ref, rtol=0, atol=1e-13)


def test_lstm_without_peepholes_is_plain_cifg_lstm():
    """With zero peepholes the ParaLSTM is torch's LSTMCell (input gate = 1 - forget)."""
    H = 4
    m, xp, prm, h0 = _rand_model("lstm", B=2, T=30, H=H, seed=2, peep=False)
    cell = torch.nn.LSTMCell(3 * H, H, dtype=f64)
    a = torch.tensor(prm["a"])
    I, Z = torch.eye(H, dtype=f64), torch.zeros(H, H, dtype=f64)
    with torch.no_grad():
        cell.weight_ih.copy_(torch.cat([torch.cat([-I, Z, Z], 1), torch.cat([I, Z, Z], 1),
                                        torch.cat([Z, I, Z], 1), torch.cat([Z, Z, I], 1)], 0))
        cell.weight_hh.copy_(torch.cat([-torch.diag(a[0]), torch.diag(a[0]), torch.diag(a[1]),
                                        torch.diag(a[2])], 0))
        cell.bias_ih.zero_()
        cell.bias_hh.zero_()
        h = torch.tensor(h0[..., 1])
        c = torch.tensor(h0[..., 0])
        outs = []
        for t in range(xp.shape[1]):
            h, c = cell(torch.tensor(xp[:, t]).reshape(2, -1), (h, c))
            outs.append(torch.stack([c, h], -1))
    np.testing.assert_allclose(m.rollout(h0), torch.stack(outs, 1).numpy(), atol=1e-13)


@pytest.mark.parametrize("cell", CELLS)
def test_step_jacobian_matches_autograd(cell):
    H = 4
    m, xp, prm, h0 = _rand_model(cell, B=2, T=5, H=H, seed=3)
    lib = _lib(cell, H, prm)
    rng = np.random.default_rng(7)
    for b, t in [(0, 0), (1, 3), (0, 4)]:
        hp = rng.standard_normal(m.h0_shape[1:])
        f, J = m.step(b, t, hp)
        p = torch.tensor(xp[b:b + 1, t])
        fn = lambda v: lib.step(p, v.reshape((1,) + hp.shape)).reshape(-1)
        hv = torch.tensor(hp).reshape(-1)
        np.testing.assert_allclose(f, fn(hv).detach().numpy(), atol=1e-13)
        Jref = torch.autograd.functional.jacobian(fn, hv).numpy()
        np.testing.assert_allclose(J, Jref, atol=1e-12)


def test_quasi_step_jacobian_is_diagonal_of_full():
    n = 6
    m, xp, prm, h0 = _rand_model("tanh", B=1, T=3, H=n, seed=4)
    mq = oracle.Model("tanh", xp, A=prm["A"], quasi=True)
    hp = np.random.default_rng(0).standard_normal(n)
    lib = _lib("tanh", n, prm)
    Jref = torch.autograd.functional.jacobian(
        lambda v: lib.step(torch.tensor(xp[0:1, 1]), v[None])[0], torch.tensor(hp)).numpy()
    f, Jq = mq.step(0, 1, hp)
    np.testing.assert_allclose(Jq, np.diag(np.diag(Jref)), atol=1e-13)


# ------------------------------------------------------------------ linear recurrences
def _dense_blocks(kind, J):
    if kind == "diag":
        return np.einsum("btn,nm->btnm", J, np.eye(J.shape[-1]))
    if kind == "block2":
        B, T, N = J.shape[:3]
        D = 2 * N
        out = np.zeros((B, T, D, D))
        for n in range(N):
            out[:, :, 2 * n:2 * n + 2, 2 * n:2 * n + 2] = J[:, :, n]
        return out
    return J


def _solve_stacked(kind, J, b, c0, reverse):
    """Dense solve of the block bidiagonal system the recurrence defines."""
    B, T = b.shape[:2]
    Jd = _dense_blocks(kind, J)
    D = Jd.shape[-1]
    bb = b.reshape(B, T, D)
    c = np.zeros((B, D)) if c0 is None else c0.reshape(B, D)
    out = np.zeros((B, T, D))
    for bi in range(B):
        M = np.eye(T * D)
        rhs = bb[bi].reshape(-1).copy()
        if not reverse:
            for t in range(1, T):
                M[t * D:(t + 1) * D, (t - 1) * D:t * D] = -Jd[bi, t]
            rhs[:D] += Jd[bi, 0] @ c[bi]
        else:
            for t in range(T - 1):
                M[t * D:(t + 1) * D, (t + 1) * D:(t + 2) * D] = -Jd[bi, t + 1].T
            rhs[(T - 1) * D:] += c[bi]
        out[bi] = np.linalg.solve(M, rhs).reshape(T, D)
    return out.reshape(b.shape)


@pytest.mark.parametrize("kind", ["diag", "block2", "dense"])
@pytest.mark.parametrize("reverse", [False, True])
@pytest.mark.parametrize("with_c0", [False, True])
def test_linear_scan_matches_dense_solve(kind, reverse, with_c0):
    rng = np.random.default_rng(11)
    B, T, N = 2, 9, 3
    if kind == "diag":
        J = rng.uniform(-1, 1, (B, T, N)); b = rng.standard_normal((B, T, N)); c0s = (B, N)
    elif kind == "block2":
        J = rng.uniform(-1, 1, (B, T, N, 2, 2)); b = rng.standard_normal((B, T, N, 2)); c0s = (B, N, 2)
    else:
        J = rng.uniform(-0.6, 0.6, (B, T, N, N)); b = rng.standard_normal((B, T, N)); c0s = (B, N)
    c0 = rng.standard_normal(c0s) if with_c0 else None
    out = oracle.linear_scan(kind, J, b, c0, reverse=reverse)
    np.testing.assert_allclose(out, _solve_stacked(kind, J, b, c0, reverse), atol=1e-12)


def test_scalar_recurrence_closed_form():
    """h_t = a h_{t-1} + b with constant a, b: h_t = a^t h0 + b (1 - a^t) / (1 - a)."""
    T, a, b, h0 = 50, 0.93, -0.37, 1.7
    out = oracle.linear_scan("diag", np.full((1, T, 1), a), np.full((1, T, 1), b),
                             np.array([[h0]]))[0, :, 0]
    t = np.arange(1, T + 1)
    np.testing.assert_allclose(out, a ** t * h0 + b * (1 - a ** t) / (1 - a), rtol=1e-13)


def test_scalar_recurrence_product_sum_form():
    """General H = 1: h_t = (prod_{s<=t} a_s) h0 + sum_s (prod_{s<r<=t} a_r) b_s."""
    rng = np.random.default_rng(5)
    T = 25
    a, b, h0 = rng.uniform(-1.2, 1.2, T), rng.standard_normal(T), 0.8
    out = oracle.linear_scan("diag", a[None, :, None], b[None, :, None], np.array([[h0]]))[0, :, 0]
    for t in range(T):
        ref = np.prod(a[: t + 1]) * h0 + sum(np.prod(a[s + 1: t + 1]) * b[s] for s in range(t + 1))
        assert abs(out[t] - ref) < 1e-12


@pytest.mark.parametrize("kind", ["diag", "block2", "dense"])
def test_reverse_scan_is_transpose_of_forward(kind):
    """<g, S b> = <S^T g, b>: the reverse (adjoint) scan is the transposed operator."""
    rng = np.random.default_rng(12)
    B, T, N = 2, 17, 3
    shp = {"diag": ((B, T, N), (B, T, N)), "block2": ((B, T, N, 2, 2), (B, T, N, 2)),
           "dense": ((B, T, N, N), (B, T, N))}[kind]
    J = rng.uniform(-0.7, 0.7, shp[0])
    b, g = rng.standard_normal(shp[1]), rng.standard_normal(shp[1])
    lhs = np.sum(g * oracle.linear_scan(kind, J, b))
    rhs = np.sum(oracle.linear_scan(kind, J, g, reverse=True) * b)
    assert abs(lhs - rhs) < 1e-11 * max(1.0, abs(lhs))


# ------------------------------------------------------------------------- Newton
@pytest.mark.parametrize("cell,quasi", [("gru", False), ("lstm", False), ("tanh", False),
                                        ("tanh", True), ("lstm", True)])
def test_newton_iterates_match_stacked_system_solve(cell, quasi):
    H = 3
    m, xp, prm, h0 = _rand_model(cell, B=2, T=7, H=H, seed=21, quasi=quasi)
    lib = _lib(cell, H, prm)
    refs = tc.newton_stacked(lib, torch.tensor(xp), torch.tensor(h0), iters=3, quasi=quasi,
                             state_shape=m.state_shape)
    for k, ref in enumerate(refs, start=1):
        h, iters, _ = m.newton(h0, max_iters=k, tol=0.0)
        assert iters == k
        np.testing.assert_allclose(h, ref.numpy(), atol=1e-11)


@pytest.mark.parametrize("cell,quasi", [("gru", False), ("lstm", False), ("tanh", False),
                                        ("tanh", True), ("lstm", True)])
def test_newton_exact_prefix_and_fixed_point(cell, quasi):
    """After k updates h_1..h_k equal the rollout; the fixed point is the rollout."""
    T = 14
    m, xp, prm, h0 = _rand_model(cell, B=2, T=T, H=4, seed=31, quasi=quasi, scale=1.5)
    R = m.rollout(h0)
    for k in range(1, T + 1):
        h, iters, _ = m.newton(h0, max_iters=k, tol=0.0)
        np.testing.assert_allclose(h[:, :k], R[:, :k], atol=1e-12)
    h, iters, deltas = m.newton(h0, max_iters=T + 1, tol=1e-12)
    assert iters <= T + 1
    np.testing.assert_allclose(h, R, atol=1e-11)
    assert deltas[-1] < 1e-12


@pytest.mark.parametrize("cell", ["gru", "tanh"])
def test_affine_cell_converges_in_one_update(cell):
    """Zero recurrent weights make the step map affine (here: constant / linear in h):
    the first update is exact and the second has delta = 0, so iters = 2."""
    B, T, H = 2, 33, 5
    rng = np.random.default_rng(41)
    G = 1 if cell == "tanh" else 3
    xp = rng.standard_normal((B, T, G, H))
    if cell == "gru":
        m = oracle.Model("gru", xp, a=np.zeros((3, H)))
    else:
        m = oracle.Model("tanh", xp, A=np.zeros((H, H)))
    h0 = rng.standard_normal((B, H))
    h, iters, deltas = m.newton(h0, max_iters=T, tol=1e-12)
    assert iters == 2
    assert deltas[1] < 1e-14
    np.testing.assert_allclose(h, m.rollout(h0), atol=1e-13)


def test_deer_with_diagonal_A_equals_quasi():
    B, T, n = 2, 20, 5
    rng = np.random.default_rng(51)
    xp = rng.standard_normal((B, T, 1, n))
    A = np.diag(rng.uniform(-0.9, 0.9, n))
    h1, i1, d1 = oracle.Model("tanh", xp, A=A).newton(max_iters=T, tol=1e-13)
    h2, i2, d2 = oracle.Model("tanh", xp, A=A, quasi=True).newton(max_iters=T, tol=1e-13)
    assert i1 == i2
    np.testing.assert_allclose(h1, h2, atol=1e-14)
    np.testing.assert_allclose(d1, d2, atol=1e-14)


def test_newton_converges_quadratically():
    """Near the solution delta_{k+1} <= C delta_k^2 with a moderate C."""
    w = wl.WORKLOADS["gru_b1_t1024_in4_h8"].resized(T=256)
    m = oracle.model_from_inputs("gru", wl.generate(w))
    _, iters, d = m.newton(max_iters=256, tol=1e-14)
    ratios = [d[k + 1] / d[k] ** 2 for k in range(len(d) - 1) if 1e-9 < d[k] < 1e-2]
    assert ratios and max(ratios) < 100.0


def test_quasi_needs_at_least_as_many_iterations_as_deer():
    w = wl.WORKLOADS["tanh_b16_t65536_in4_n8_deer"].resized(B=2, T=512)
    inp = wl.generate(w)
    _, i_full, _ = oracle.model_from_inputs("tanh", inp).newton(max_iters=512, tol=1e-5)
    _, i_quasi, _ = oracle.model_from_inputs("tanh", inp, quasi=True).newton(max_iters=512, tol=1e-5)
    assert i_quasi >= i_full


def test_quasi_lstm_needs_at_least_as_many_iterations_as_block_newton():
    """The diagonal (quasi) backend drops the c-h coupling of each 2x2 block: same
    fixed point, no faster convergence."""
    w = wl.WORKLOADS["lstm_b4_t8192_h1024_bf16"].resized(B=2, T=256, H=16, inp=16, bf16=False)
    inp = wl.generate(w)
    h_b, i_b, _ = oracle.model_from_inputs("lstm", inp).newton(max_iters=256, tol=1e-9)
    h_q, i_q, _ = oracle.model_from_inputs("lstm", inp, quasi=True).newton(max_iters=256, tol=1e-9)
    assert i_q >= i_b
    np.testing.assert_allclose(h_q, h_b, atol=1e-8)


def _fixed_point_sweeps(lib, xp, h0, iters, solver):
    """Jacobi: h^(k+1)_t = f(h^(k)_{t-1}); Picard: h^(k+1)_t = h^(k+1)_{t-1} +
    f(h^(k)_{t-1}) - h^(k)_{t-1}; both from h^(0) = 0, with the library cell."""
    xpt, h0t = torch.tensor(xp), torch.tensor(h0)
    B, T = xp.shape[:2]
    hs = torch.zeros((B, T) + tuple(h0t.shape[1:]), dtype=f64)
    for _ in range(iters):
        prev = torch.cat([h0t[:, None], hs[:, :-1]], 1)
        f = torch.stack([lib.step(xpt[:, t], prev[:, t]) for t in range(T)], 1)
        if solver == "jacobi":
            hs = f
        else:
            inc = f - prev
            new, acc = [], h0t
            for t in range(T):
                acc = acc + inc[:, t]
                new.append(acc)
            hs = torch.stack(new, 1)
    return hs.numpy()


@pytest.mark.parametrize("cell", CELLS)
@pytest.mark.parametrize("solver", ["jacobi", "picard"])
def test_fixed_point_sweeps_match_their_definition(cell, solver):
    """The Jacobi (J = 0) and Picard (J = I) linearisations in the Newton loop equal the
    sweeps written out with the library cell, and keep the exact-prefix property."""
    H, T = 3, 9
    m, xp, prm, h0 = _rand_model(cell, B=2, T=T, H=H, seed=61)
    m = oracle.Model(cell, xp, solver=solver, **prm)
    lib = _lib(cell, H, prm)
    R = m.rollout(h0)
    for k in (1, 2, 5):
        h, iters, _ = m.newton(h0, max_iters=k, tol=0.0)
        assert iters == k
        np.testing.assert_allclose(h, _fixed_point_sweeps(lib, xp, h0, k, solver), atol=1e-12)
        np.testing.assert_allclose(h[:, :k], R[:, :k], atol=1e-12)
    h, iters, _ = m.newton(h0, max_iters=T + 1, tol=1e-13)
    np.testing.assert_allclose(h, R, atol=1e-12)


def _lm_stacked(lib, xp, h0, iters, lam, state_shape, diag_only=True):
    """Levenberg-Marquardt on the stacked residual F(h) = 0 with a dense solve:
    h <- h - (Jd^T Jd + lam I)^{-1} Jd^T F, where Jd is dF/dh (autograd), with only the
    diagonal of each sub-diagonal block kept (the diagonal linearisation) when
    diag_only, else the whole Jacobian (full 2x2 blocks for the LSTM)."""
    xpt, h0t = torch.tensor(xp), torch.tensor(h0)
    hs = torch.zeros(state_shape, dtype=f64)
    B, T = hs.shape[:2]
    D = hs[0, 0].numel()
    out = []
    for _ in range(iters):
        F = tc.stacked_residual(lib, xpt, h0t, hs).reshape(-1)
        Jf = torch.autograd.functional.jacobian(
            lambda v: tc.stacked_residual(lib, xpt, h0t, v.reshape(hs.shape)).reshape(-1), hs.reshape(-1))
        Jm = Jf.reshape(B, T, D, B, T, D).clone()
        if diag_only:
            off = ~torch.eye(D, dtype=torch.bool)
            for b in range(B):
                for t in range(1, T):
                    blk = Jm[b, t, :, b, t - 1, :]
                    blk[off] = 0.0
        Jd = Jm.reshape(B * T * D, B * T * D)
        step = torch.linalg.solve(Jd.T @ Jd + lam * torch.eye(Jd.shape[0], dtype=f64), Jd.T @ F)
        hs = hs - step.reshape(hs.shape)
        out.append(hs.clone())
    return out


ELK_VARIANTS = [("gru", False), ("lstm", False), ("lstm", True), ("tanh", False)]


@pytest.mark.parametrize("cell,quasi", ELK_VARIANTS)
@pytest.mark.parametrize("lam", [0.3, 2.0])
def test_elk_step_is_levenberg_marquardt_on_stacked_system(cell, quasi, lam):
    """The Kalman-smoother step equals the dense Levenberg-Marquardt step: with the
    LSTM's full 2x2 blocks (ELK), or each block's diagonal (quasi-ELK; the tanh RNN's
    ELK always takes the diagonal of its dense Jacobian)."""
    H = 3
    m, xp, prm, h0 = _rand_model(cell, B=2, T=8, H=H, seed=71)
    m = oracle.Model(cell, xp, solver="elk", damping=lam, quasi=quasi, **prm)
    full = cell == "lstm" and not quasi
    refs = _lm_stacked(_lib(cell, H, prm), xp, h0, 3, lam, m.state_shape, diag_only=not full)
    for k, ref in enumerate(refs, start=1):
        h, iters, _ = m.newton(h0, max_iters=k, tol=0.0)
        assert iters == k
        np.testing.assert_allclose(h, ref.numpy(), atol=1e-11)


@pytest.mark.parametrize("cell,quasi", ELK_VARIANTS)
def test_elk_without_damping_is_the_newton_step(cell, quasi):
    """lambda = 0: the step of the same linearisation without damping (the full-block
    Newton step for ELK on the LSTM, the diagonal quasi-Newton step otherwise)."""
    m, xp, prm, h0 = _rand_model(cell, B=2, T=30, H=4, seed=72)
    e = oracle.Model(cell, xp, solver="elk", damping=0.0, quasi=quasi, **prm)
    q = oracle.Model(cell, xp, quasi=quasi or cell == "tanh", **prm)  # GRU: its Jacobian is already diagonal
    for k in (1, 2, 4):
        np.testing.assert_allclose(e.newton(h0, max_iters=k, tol=0.0)[0], q.newton(h0, max_iters=k, tol=0.0)[0],
                                   atol=1e-12)


@pytest.mark.parametrize("cell,quasi", ELK_VARIANTS)
def test_elk_converges_to_rollout_and_damping_shortens_steps(cell, quasi):
    m, xp, prm, h0 = _rand_model(cell, B=2, T=40, H=4, seed=73, scale=1.5)
    R = m.rollout(h0)
    h, iters, d = oracle.Model(cell, xp, solver="elk", damping=0.5, quasi=quasi, **prm).newton(
        h0, max_iters=400, tol=1e-12)
    np.testing.assert_allclose(h, R, atol=1e-10)
    first = [oracle.Model(cell, xp, solver="elk", damping=lam, quasi=quasi, **prm).newton(
        h0, max_iters=1, tol=0.0)[2][0] for lam in (0.0, 0.5, 5.0)]
    assert first[0] > first[1] > first[2]


def _block_lm_dense(J, r, lam):
    """argmin_x sum_t |x_t - J_t x_{t-1} - r_t|^2 + lam |x|^2 (x_{-1} = 0), solved densely."""
    T = J.shape[0]
    L = np.eye(2 * T)
    for t in range(1, T):
        L[2 * t:2 * t + 2, 2 * t - 2:2 * t] = -J[t]
    return np.linalg.solve(L.T @ L + lam * np.eye(2 * T), L.T @ r.reshape(-1)).reshape(T, 2)


@pytest.mark.parametrize("T", [1, 7, 40])
@pytest.mark.parametrize("lam", [0.0, 0.4, 3.0])
def test_block_smoother_is_the_dense_lm_solution(T, lam):
    """The 2x2 Kalman filter + RTS smoother against the normal equations of its objective."""
    rng = np.random.default_rng(T * 10 + int(lam * 10))
    J = rng.standard_normal((T, 2, 2)) * 0.8
    r = rng.standard_normal((T, 2))
    np.testing.assert_allclose(oracle.elk_block2(J, r, lam), _block_lm_dense(J, r, lam), atol=1e-11)


def test_block_smoother_without_damping_is_the_forward_recursion():
    rng = np.random.default_rng(5)
    T = 50
    J = rng.standard_normal((T, 2, 2)) * 0.5
    r = rng.standard_normal((T, 2))
    x, ref = np.zeros(2), []
    for t in range(T):
        x = J[t] @ x + r[t]
        ref.append(x)
    np.testing.assert_allclose(oracle.elk_block2(J, r, 0.0), np.array(ref), atol=1e-12)


def test_block_smoother_with_diagonal_blocks_is_two_scalar_smoothers():
    rng = np.random.default_rng(6)
    T = 60
    a = rng.uniform(-1.2, 1.2, (T, 2))
    r = rng.standard_normal((T, 2))
    J = np.zeros((T, 2, 2))
    J[:, 0, 0], J[:, 1, 1] = a[:, 0], a[:, 1]
    x = oracle.elk_block2(J, r, 0.8)
    for s in range(2):
        np.testing.assert_allclose(x[:, s], oracle.elk_scalar(a[:, s], r[:, s], 0.8), atol=1e-12)


def test_scalar_smoother_is_the_dense_lm_solution():
    rng = np.random.default_rng(7)
    T = 30
    a, r = rng.uniform(-1.5, 1.5, T), rng.standard_normal(T)
    L = np.eye(T) - np.diag(a[1:], -1)
    ref = np.linalg.solve(L.T @ L + 1.3 * np.eye(T), L.T @ r)
    np.testing.assert_allclose(oracle.elk_scalar(a, r, 1.3), ref, atol=1e-12)


def test_newton_zero_iterations_returns_initial_guess():
    m, xp, prm, h0 = _rand_model("gru", B=1, T=5, H=2, seed=3)
    h, iters, d = m.newton(h0, max_iters=0, tol=1e-6)
    assert iters == 0 and np.all(h == 0)


# ------------------------------------------------------------------------- adjoint
def _adjoint_ref_implicit(cell, m, xp, prm, h0, h, g):
    """lambda = (dF/dh)^{-T} g; grads = -(dF/dtheta)^T lambda (autograd + dense solve)."""
    H = m.H
    lib = _lib(cell, H, prm)
    xpt = torch.tensor(xp, requires_grad=True)
    a = torch.tensor(prm["a"], requires_grad=True)
    peep = torch.tensor(prm["peep"], requires_grad=True) if cell == "lstm" else None
    h0t = torch.tensor(h0, requires_grad=True)
    hs = torch.tensor(h)
    kw = {"a": a} if cell == "gru" else {"a": a, "peep": peep}
    kw_const = {k: x.detach() for k, x in kw.items()}
    Jf = torch.autograd.functional.jacobian(
        lambda v: tc.stacked_residual(lib, xpt.detach(), h0t.detach(), v.reshape(hs.shape),
                                      **kw_const).reshape(-1),
        hs.reshape(-1))
    lam = torch.linalg.solve(Jf.T, torch.tensor(g).reshape(-1))
    F = tc.stacked_residual(lib, xpt, h0t, hs, **kw).reshape(-1)
    params = [xpt, a] + ([peep] if cell == "lstm" else []) + [h0t]
    grads = torch.autograd.grad(F, params, grad_outputs=-lam)
    gx, ga = grads[0].numpy(), grads[1].numpy()
    gpe = grads[2].numpy() if cell == "lstm" else None
    gh0 = grads[-1].numpy()
    gp = ga if cell == "gru" else np.concatenate([ga, gpe], 0)
    return gx, gp, gh0


@pytest.mark.parametrize("cell", ["gru", "lstm"])
def test_adjoint_matches_autograd_through_rollout(cell):
    H = 3
    m, xp, prm, h0 = _rand_model(cell, B=2, T=12, H=H, seed=61)
    rng = np.random.default_rng(62)
    g = rng.standard_normal(m.state_shape)
    h = m.rollout(h0)
    gx, gp, gh0 = m.adjoint(h, g, h0)
    lib = _lib(cell, H, prm)
    xpt = torch.tensor(xp, requires_grad=True)
    a = torch.tensor(prm["a"], requires_grad=True)
    peep = torch.tensor(prm["peep"], requires_grad=True) if cell == "lstm" else None
    h0t = torch.tensor(h0, requires_grad=True)
    hs, hcur = [], h0t
    for t in range(xp.shape[1]):
        hcur = lib.step(xpt[:, t], hcur, a=a) if cell == "gru" else lib.step(xpt[:, t], hcur, a=a, peep=peep)
        hs.append(hcur)
    L = (torch.stack(hs, 1) * torch.tensor(g)).sum()
    params = [xpt, a] + ([peep] if cell == "lstm" else []) + [h0t]
    grads = torch.autograd.grad(L, params)
    np.testing.assert_allclose(gx, grads[0].numpy(), atol=1e-11)
    ref_gp = grads[1].numpy() if cell == "gru" else np.concatenate([grads[1].numpy(), grads[2].numpy()])
    np.testing.assert_allclose(gp, ref_gp, atol=1e-10)
    np.testing.assert_allclose(gh0, grads[-1].numpy(), atol=1e-11)


@pytest.mark.parametrize("cell", ["gru", "lstm"])
def test_adjoint_at_unconverged_states_is_implicit_gradient(cell):
    """At any states (e.g. 2 Newton updates), the adjoint is the implicit-function
    gradient with every Jacobian evaluated at those states."""
    H = 3
    m, xp, prm, h0 = _rand_model(cell, B=2, T=10, H=H, seed=71, scale=1.5)
    h, _, _ = m.newton(h0, max_iters=2, tol=0.0)
    g = np.random.default_rng(72).standard_normal(m.state_shape)
    gx, gp, gh0 = m.adjoint(h, g, h0)
    rx, rp, rh0 = _adjoint_ref_implicit(cell, m, xp, prm, h0, h, g)
    np.testing.assert_allclose(gx, rx, atol=1e-10)
    np.testing.assert_allclose(gp, rp, atol=1e-10)
    np.testing.assert_allclose(gh0, rh0, atol=1e-10)


# ------------------------------------------------------------------------- residual
@pytest.mark.parametrize("cell", CELLS)
def test_residual_matches_library_step(cell):
    H = 4
    m, xp, prm, h0 = _rand_model(cell, B=2, T=9, H=H, seed=81)
    h, _, _ = m.newton(h0, max_iters=3, tol=0.0)
    lib = _lib(cell, H, prm)
    F = tc.stacked_residual(lib, torch.tensor(xp), torch.tensor(h0), torch.tensor(h))
    assert abs(m.residual(h, h0) - F.abs().max().item()) < 1e-13
    assert m.residual(m.rollout(h0), h0) < 1e-14


# ------------------------------------------------------------------------- projection
def test_input_proj_matches_brute_force():
    rng = np.random.default_rng(91)
    x = wl.round_bf16(rng.standard_normal((2, 3, 5)).astype(np.float32))
    W = wl.round_bf16(rng.standard_normal((4, 5)).astype(np.float32))
    bias = rng.standard_normal(4).astype(np.float32)
    y = oracle.input_proj(x, W, bias)
    for b in range(2):
        for t in range(3):
            for n in range(4):
                ref = float(bias[n]) + sum(float(x[b, t, k]) * float(W[n, k]) for k in range(5))
                assert abs(y[b, t, n] - ref) < 1e-12


def test_input_proj_backward_matches_brute_force_sums():
    rng = np.random.default_rng(92)
    M, K, N = 5, 4, 3
    g = rng.standard_normal((M, N))
    x = rng.standard_normal((M, K))
    W = rng.standard_normal((N, K))
    gx, gW, gb = oracle.input_proj_backward(g, x, W)
    for m in range(M):
        for k in range(K):
            assert abs(gx[m, k] - sum(g[m, n] * W[n, k] for n in range(N))) < 1e-12
    for n in range(N):
        for k in range(K):
            assert abs(gW[n, k] - sum(g[m, n] * x[m, k] for m in range(M))) < 1e-12
        assert abs(gb[n] - sum(g[m, n] for m in range(M))) < 1e-12


def test_input_proj_backward_matches_autograd_of_library_linear():
    """The gradients of torch.nn.functional.linear (a library layer, autograd)."""
    rng = np.random.default_rng(93)
    x = torch.tensor(rng.standard_normal((2, 3, 6)), dtype=f64, requires_grad=True)
    W = torch.tensor(rng.standard_normal((4, 6)), dtype=f64, requires_grad=True)
    bias = torch.tensor(rng.standard_normal(4), dtype=f64, requires_grad=True)
    g = rng.standard_normal((2, 3, 4))
    (torch.nn.functional.linear(x, W, bias) * torch.tensor(g)).sum().backward()
    gx, gW, gb = oracle.input_proj_backward(g, x.detach().numpy(), W.detach().numpy())
    assert np.abs(gx.reshape(2, 3, 6) - x.grad.numpy()).max() < 1e-12
    assert np.abs(gW - W.grad.numpy()).max() < 1e-12
    assert np.abs(gb - bias.grad.numpy()).max() < 1e-12


def test_input_proj_backward_adjoint_identity():
    """<g, x W^T> = <grad_W, W> = <grad_x, x> (the projection is bilinear)."""
    rng = np.random.default_rng(94)
    g = rng.standard_normal((7, 5))
    x = rng.standard_normal((7, 3))
    W = rng.standard_normal((5, 3))
    gx, gW, _ = oracle.input_proj_backward(g, x, W)
    lhs = float((g * oracle.input_proj(x, W)).sum())
    assert abs(lhs - float((gW * W).sum())) < 1e-10
    assert abs(lhs - float((gx * x).sum())) < 1e-10


def test_model_from_inputs_layout_gate_major():
    """xproj[b, t, g, u] uses W row g*H + u (gate-major), as the layout promises."""
    w = wl.WORKLOADS["gru_b1_t1024_in4_h8"].resized(T=3)
    inp = wl.generate(w)
    m = oracle.model_from_inputs("gru", inp)
    H = w.H
    for g_ in range(3):
        for u in range(H):
            ref = inp["x"][0, 2].astype(np.float64) @ inp["W"][g_ * H + u].astype(np.float64)
            assert abs(m.xproj[0, 2, g_, u] - ref - inp["bias"][g_ * H + u]) < 1e-12


def test_tolerance_test_is_strict():
    """Stop only when delta < tol: with tol = 0 an exactly converged solve (delta = 0)
    still runs to max_iters, which is how a fixed iteration count is requested."""
    B, T, H = 1, 8, 2
    xp = np.random.default_rng(3).standard_normal((B, T, 3, H))
    m = oracle.Model("gru", xp, a=np.zeros((3, H)))
    _, iters, d = m.newton(max_iters=5, tol=0.0)
    assert iters == 5 and d[1] == 0.0
    _, iters, _ = m.newton(max_iters=5, tol=1e-300)
    assert iters == 2
