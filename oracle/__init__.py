"""fp64 CPU oracle for the Newton (DEER) / quasi-Newton evaluation of nonlinear RNNs,
its fixed-point variants, the linear scans, the adjoint and the fixed-step simulation of
linear ODEs (lsim).

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline / reference leg of ``bench.py`` may import this package.  The CUDA
library never links, loads or calls it, and this package imports nothing from
the CUDA library: the two share only the seeded input generator.

The arithmetic lives in ``oracle.c`` (plain C, fp64, sequential in time, OpenMP
only over independent sequences).  This module marshals numpy arrays into it
and holds the two steps that are library primitives: the input projection
``x W^T + bias`` as a float64 numpy matmul, and the matrix exponential that
discretises a linear ODE over one step (``scipy.linalg.expm``).

Every function here is pinned by the CPU tests against something other than
itself (PyTorch's reference GRU/LSTM/RNN cells, autograd Jacobians, dense
linear solves of the stacked system, closed forms and invariants; for lsim, closed
forms, exact quadrature sums, an RK4 integration and scipy's own lsim).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

CELL_IDS = {"gru": 0, "lstm": 1, "tanh": 2}
SCAN_IDS = {"diag": 0, "block2": 1, "dense": 2}


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so next to it (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


class _Model(ctypes.Structure):
    _fields_ = [("cell", ctypes.c_int), ("quasi", ctypes.c_int),
                ("B", ctypes.c_long), ("T", ctypes.c_long), ("H", ctypes.c_long),
                ("xproj", ctypes.c_void_p), ("a", ctypes.c_void_p),
                ("peep", ctypes.c_void_p), ("A", ctypes.c_void_p), ("solver", ctypes.c_int),
                ("lambda_", ctypes.c_double)]


_lib = None


def _L():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        _lib.orc_residual.restype = ctypes.c_double
        _lib.orc_get_threads.restype = ctypes.c_int
    return _lib


def _f64(a):
    if a is None:
        return None
    return np.ascontiguousarray(np.asarray(a), dtype=np.float64)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def set_threads(n: int) -> None:
    _L().orc_set_threads(int(n))


def get_threads() -> int:
    return int(_L().orc_get_threads())


def elk_block2(J, r, lam):
    """The damped step of one unit with 2x2 Jacobian blocks (Kalman filter + RTS smoother
    in oracle.c): J [T, 2, 2], r [T, 2] -> x [T, 2]."""
    J = _f64(J).reshape(-1, 4)
    r = _f64(r).reshape(-1, 2)
    T = J.shape[0]
    xs = np.zeros((T, 2))
    rc = _L().orc_elk_block2(ctypes.c_long(T), _ptr(J), _ptr(r), ctypes.c_double(float(lam)), _ptr(xs))
    assert rc == 0
    return xs


def elk_scalar(a, r, lam):
    """The damped step of one scalar component (Kalman filter + RTS smoother in oracle.c):
    a [T], r [T] -> x [T]."""
    a, r = _f64(a).ravel(), _f64(r).ravel()
    xs = np.zeros(a.shape[0])
    rc = _L().orc_elk_scalar(ctypes.c_long(a.shape[0]), _ptr(a), _ptr(r), ctypes.c_double(float(lam)), _ptr(xs))
    assert rc == 0
    return xs


class Model:
    """Cell + parameters + projected inputs, all widened exactly to float64.

    xproj: [B, T, G, H] (G = 3 GRU/LSTM, 1 tanh), a: [3, H], peep: [2, H], A: [n, n].
    """

    SOLVERS = {"newton": 0, "jacobi": 1, "picard": 2, "elk": 3}

    def __init__(self, cell, xproj, a=None, peep=None, A=None, quasi=False, solver="newton",
                 damping=0.0):
        self.cell = cell
        self.xproj = _f64(xproj)
        B, T, G, H = self.xproj.shape
        assert G == (1 if cell == "tanh" else 3)
        self.B, self.T, self.H = B, T, H
        self.a, self.peep, self.A = _f64(a), _f64(peep), _f64(A)
        self.quasi = bool(quasi)
        self.S = 2 if cell == "lstm" else 1
        self.solver = solver
        self.damping = float(damping)
        self._m = _Model(CELL_IDS[cell], int(self.quasi), B, T, H, _ptr(self.xproj),
                         _ptr(self.a), _ptr(self.peep), _ptr(self.A), self.SOLVERS[solver],
                         self.damping)

    @property
    def state_shape(self):
        return (self.B, self.T, self.H, 2) if self.cell == "lstm" else (self.B, self.T, self.H)

    @property
    def h0_shape(self):
        return (self.B, self.H, 2) if self.cell == "lstm" else (self.B, self.H)

    def _h0(self, h0):
        if h0 is None:
            return None
        h0 = _f64(h0)
        assert h0.shape == self.h0_shape
        return h0

    def rollout(self, h0=None):
        """Sequential h_t = f(h_{t-1}, x_t)."""
        h0 = self._h0(h0)
        h = np.zeros(self.state_shape)
        _L().orc_rollout(ctypes.byref(self._m), _ptr(h0), _ptr(h))
        return h

    def newton(self, h0=None, max_iters=None, tol=0.0, log_len=None):
        """Newton / quasi-Newton solve from h^(0) = 0.  Returns (h, iters, deltas)."""
        h0 = self._h0(h0)
        if max_iters is None:
            max_iters = self.T
        log_len = max_iters if log_len is None else log_len
        h = np.zeros(self.state_shape)
        deltas = np.zeros(max(log_len, 1))
        iters = ctypes.c_int(0)
        rc = _L().orc_newton(ctypes.byref(self._m), _ptr(h0), ctypes.c_int(int(max_iters)),
                             ctypes.c_double(float(tol)), _ptr(h), ctypes.byref(iters),
                             _ptr(deltas), ctypes.c_int(int(log_len)))
        assert rc == 0
        return h, int(iters.value), deltas[: min(int(iters.value), log_len)].copy()

    def step(self, b, t, hp):
        """f and the full Jacobian of the step map at (b, t) from state vector hp."""
        D = self.H * self.S if self.cell != "tanh" else self.H
        hp = _f64(hp).reshape(D)
        f = np.zeros(D)
        J = np.zeros((D, D))
        _L().orc_step(ctypes.byref(self._m), ctypes.c_long(b), ctypes.c_long(t), _ptr(hp),
                      _ptr(f), _ptr(J))
        return f, J

    def adjoint(self, h, g, h0=None):
        """Adjoint gradients of L = sum <g, h> at states h (GRU/LSTM).

        Returns (grad_xproj [B,T,3,H], grad_params [3 or 5, H], grad_h0 [h0 shape]).
        """
        assert self.cell in ("gru", "lstm")
        h0 = self._h0(h0)
        h, g = _f64(h), _f64(g)
        assert h.shape == self.state_shape and g.shape == self.state_shape
        gx = np.zeros((self.B, self.T, 3, self.H))
        gp = np.zeros((3 if self.cell == "gru" else 5, self.H))
        gh0 = np.zeros(self.h0_shape)
        rc = _L().orc_adjoint(ctypes.byref(self._m), _ptr(h0), _ptr(h), _ptr(g), _ptr(gx),
                              _ptr(gp), _ptr(gh0))
        assert rc == 0
        return gx, gp, gh0

    def residual(self, h, h0=None):
        """max |h_t - f(h_{t-1}, x_t)| over every state element."""
        h0 = self._h0(h0)
        h = _f64(h)
        return float(_L().orc_residual(ctypes.byref(self._m), _ptr(h0), _ptr(h)))


def input_proj(x, W, bias=None):
    """xproj = x W^T + bias in float64 (a library matmul), x [..., in], W [N, in]."""
    x64, W64 = _f64(x), _f64(W)
    y = x64.reshape(-1, x64.shape[-1]) @ W64.T
    if bias is not None:
        y = y + _f64(bias)[None, :]
    return y.reshape(*x64.shape[:-1], W64.shape[0])


def input_proj_backward(grad_xproj, x, W):
    """Gradients of L = <grad_xproj, x W^T + bias> (float64 library matmuls).

    The projection is linear in x, W and bias, so its reverse pass is three plain
    contractions ("Para-Seq" README, Main features: trainable GRU/LSTM layers whose
    input projection precedes the parallel solve):
      grad_x    [M, K] = grad_xproj [M, N] @ W [N, K]
      grad_W    [N, K] = grad_xproj^T @ x [M, K]
      grad_bias [N]    = column sums of grad_xproj
    Leading dimensions of grad_xproj and x are flattened to M.
    """
    g64, x64, W64 = _f64(grad_xproj), _f64(x), _f64(W)
    g2 = g64.reshape(-1, g64.shape[-1])
    x2 = x64.reshape(-1, x64.shape[-1])
    return g2 @ W64, g2.T @ x2, g2.sum(axis=0)


def model_from_inputs(cell, inputs, quasi=False, solver="newton", damping=0.0):
    """Build a Model from the arrays of ``workloads.generate`` (projection in fp64)."""
    x = inputs["x"]
    B, T, _ = x.shape
    xp = input_proj(x, inputs["W"], inputs.get("bias"))
    G = 1 if cell == "tanh" else 3
    H = xp.shape[-1] // G
    xp = xp.reshape(B, T, G, H)
    return Model(cell, xp, a=inputs.get("a"), peep=inputs.get("peep"), A=inputs.get("A"),
                 quasi=quasi, solver=solver, damping=damping)


def linear_scan(kind, J, b, h0=None, reverse=False):
    """Sequential linear recurrence (see oracle.c).  kind: diag | block2 | dense.

    diag:   J [B,T,N],       b [B,T,N],    h0 [B,N]
    block2: J [B,T,N,2,2],   b [B,T,N,2],  h0 [B,N,2]
    dense:  J [B,T,N,N],     b [B,T,N],    h0 [B,N]
    """
    J, b = _f64(J), _f64(b)
    B, T, N = b.shape[:3]
    h0 = _f64(h0)
    out = np.zeros_like(b)
    rc = _L().orc_linear_scan(ctypes.c_int(SCAN_IDS[kind]), ctypes.c_long(B), ctypes.c_long(T),
                              ctypes.c_long(N), _ptr(J), _ptr(b), _ptr(h0), _ptr(out),
                              ctypes.c_int(int(bool(reverse))))
    assert rc == 0
    return out


LSIM_INTERP = {"zoh": 0, "foh": 1}


def lsim_discretize(A, B, h, interp="zoh"):
    """One step of the linear ODE dx/dt = A x + B u, exact for an input held constant
    over the step ("zoh") or varying linearly between samples ("foh"): returns
    (Ad, G0, G1) with x_{k+1} = Ad x_k + G0 u_k + G1 u_{k+1}.

    ("Para-Seq" README, Quick example: ``lsim(A, B, C, D, U, t)`` on a fixed-step time
    grid; the pages name no hold rule, and these are the two exact ones.)  Both come
    from one exponential of a block upper-triangular matrix (Van Loan's construction):
      zoh: expm([[A h, B h], [0, 0]])            = [[Ad, P0], [0, I]]
      foh: expm([[A h, B h, 0], [0, 0, I], [0, 0, 0]]) = [[Ad, P0, P1], [0, I, I], [0, 0, I]]
    with P0 = int_0^h e^{A s} ds B and P1 = int_0^h e^{A s} (h - s)/h ds B.  A held
    input gives G0 = P0, G1 = 0; a linear one u(t_k + s) = u_k + (s/h)(u_{k+1} - u_k)
    gives G0 = P0 - P1, G1 = P1.
    """
    import scipy.linalg

    A, B = _f64(A), _f64(B)
    n, m = B.shape
    if LSIM_INTERP[interp] == 0:
        M = np.zeros((n + m, n + m))
        M[:n, :n] = A * h
        M[:n, n:] = B * h
        E = scipy.linalg.expm(M)
        return E[:n, :n].copy(), E[:n, n:].copy(), np.zeros((n, m))
    M = np.zeros((n + 2 * m, n + 2 * m))
    M[:n, :n] = A * h
    M[:n, n:n + m] = B * h
    M[n:n + m, n + m:] = np.eye(m)
    E = scipy.linalg.expm(M)
    P0, P1 = E[:n, n:n + m], E[:n, n + m:]
    return E[:n, :n].copy(), (P0 - P1).copy(), P1.copy()


def lsim(A, B, C, D, U, h, x0=None, interp="zoh"):
    """Fixed-step linear simulation ("Para-Seq" README, Quick example): the system
    discretised by ``lsim_discretize`` and stepped sequentially in fp64 (oracle.c).

    U [T, m] or [batch, T, m]; x0 [n] or [batch, n] (zero when None).  Returns
    (y [.., T, p], x [.., T, n]): x_0 = x0, x_k = Ad x_{k-1} + G0 u_{k-1} + G1 u_k,
    y_k = C x_k + D u_k (D None: no feedthrough).
    """
    U = _f64(U)
    single = U.ndim == 2
    if single:
        U = U[None]
    Bt, T, m = U.shape
    Ad, G0, G1 = lsim_discretize(A, B, h, interp)
    n = Ad.shape[0]
    C = _f64(C)
    p = C.shape[0]
    D = None if D is None else _f64(D)
    if x0 is not None:
        x0 = np.ascontiguousarray(np.broadcast_to(_f64(x0), (Bt, n)))
    y = np.zeros((Bt, T, p))
    x = np.zeros((Bt, T, n))
    _L().orc_lti_sim(ctypes.c_long(Bt), ctypes.c_long(T), ctypes.c_int(n), ctypes.c_int(m), ctypes.c_int(p),
                     _ptr(Ad), _ptr(G0), _ptr(G1), _ptr(C), _ptr(D), _ptr(U), _ptr(x0), _ptr(y), _ptr(x))
    return (y[0], x[0]) if single else (y, x)
