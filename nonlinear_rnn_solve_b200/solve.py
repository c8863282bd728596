"""Output allocation around the C ABI (marshalling only; the work runs in libpararnn.so).

Each function allocates its outputs with torch on the inputs' device, calls one
entry point of ``include/pararnn.h`` on the context's stream, and returns tensors.
"""
from __future__ import annotations

import torch

from . import (PARARNN_GRU_DIAG, PARARNN_LSTM_CIFG_PEEP, PARARNN_RNN_TANH_DENSE,
               PARARNN_RNN_TANH_QUASI, PARARNN_LSTM_CIFG_PEEP_QUASI, make_params, pararnn_adjoint_backward,
               pararnn_input_proj, pararnn_linear_scan, pararnn_newton_forward)

CELLS = {"gru": PARARNN_GRU_DIAG, "lstm": PARARNN_LSTM_CIFG_PEEP,
         "tanh": PARARNN_RNN_TANH_DENSE, "tanh_quasi": PARARNN_RNN_TANH_QUASI,
         "lstm_quasi": PARARNN_LSTM_CIFG_PEEP_QUASI}


def state_shape(cell, B, T, H):
    return (B, T, H, 2) if cell in ("lstm", "lstm_quasi") else (B, T, H)


SOLVERS = {"newton": 0, "jacobi": 1, "picard": 2, "elk": 3}


def _need(t, count, name):
    """The C ABI takes bare pointers: check each operand's element count first."""
    if t is not None and t.numel() != count:
        raise ValueError(f"{name} has {t.numel()} elements, expected {count}")


def newton_forward(ctx, cell, B, T, H, *, xproj=None, x=None, W=None, bias=None, a=None,
                   peep=None, A=None, h0=None, max_iters=None, tol=1e-6, residual=False,
                   h_out=None, solver="newton", damping=0.0, scalars=None):
    """Newton / quasi-Newton (or Jacobi / Picard) solve.  Returns dict(h, iters, delta,
    residual) (device tensors).  ``scalars``: optional dict with preallocated one-element
    device tensors "iters" (int32), "delta" and "residual" (fp32), reused instead of
    allocating new ones (no fill launches around the solve)."""
    dev = (xproj if xproj is not None else x).device
    inp = 0 if x is None else x.shape[-1]
    G = 1 if cell in ("tanh", "tanh_quasi") else 3
    S = 2 if cell in ("lstm", "lstm_quasi") else 1
    if xproj is not None:
        _need(xproj, B * T * G * H, "xproj [B, T, G, H]")
    else:
        _need(x, B * T * inp, "x [B, T, in]")
        _need(W, G * H * inp, "W [G*H, in]")
        _need(bias, G * H, "bias [G*H]")
    if G == 3:
        _need(a, 3 * H, "a [3, H]")
        _need(peep, 2 * H, "peep [2, H]")
    else:
        _need(A, H * H, "A [n, n]")
    _need(h0, B * H * S, "h0")
    _need(h_out, B * T * H * S, "h_out")
    prm = make_params(CELLS[cell], B, T, H, inp, a=a, peep=peep, A=A,
                      x=x if xproj is None else None, W=W if xproj is None else None,
                      bias=bias if xproj is None else None, solver=SOLVERS[solver], damping=damping)
    if h_out is None:
        h_out = torch.empty(state_shape(cell, B, T, H), device=dev, dtype=torch.float32)
    if scalars is not None:
        iters, delta = scalars["iters"], scalars["delta"]
        res = scalars["residual"] if residual else None
        _need(iters, 1, "iters")
        _need(delta, 1, "delta")
        _need(res, 1, "residual")
    else:
        iters = torch.zeros(1, device=dev, dtype=torch.int32)
        delta = torch.zeros(1, device=dev, dtype=torch.float32)
        res = torch.zeros(1, device=dev, dtype=torch.float32) if residual else None
    pararnn_newton_forward(ctx, xproj, prm, h0, h_out, T if max_iters is None else max_iters, tol,
                           iters, delta, res)
    return {"h": h_out, "iters": iters, "delta": delta, "residual": res}


def input_proj(ctx, x, W, bias=None):
    """xproj = x W^T + bias with x [..., K] and W [N, K] (both bf16 or both fp32)."""
    N = W.shape[0]
    _need(W, N * x.shape[-1], "W [N, K]")
    _need(bias, N, "bias [N]")
    out = torch.empty(*x.shape[:-1], N, device=x.device, dtype=torch.float32)
    pararnn_input_proj(ctx, x, W, bias, out)
    return out


def input_proj_backward(ctx, grad_xproj, x, W, need_x=True, need_W=True, need_bias=True):
    """Gradients of the projection: (grad_x [..., K], grad_W [N, K], grad_bias [N]);
    entries not requested are None."""
    from . import pararnn_input_proj_backward
    dev = x.device
    K, N = x.shape[-1], W.shape[0]
    _need(W, N * K, "W [N, K]")
    _need(grad_xproj, (x.numel() // K) * N, "grad_xproj [M, N]")
    gx = torch.empty(*x.shape[:-1], K, device=dev, dtype=torch.float32) if need_x else None
    gW = torch.empty(N, K, device=dev, dtype=torch.float32) if need_W else None
    gb = torch.empty(N, device=dev, dtype=torch.float32) if need_bias else None
    pararnn_input_proj_backward(ctx, grad_xproj, x, W, gx, gW, gb)
    return gx, gW, gb


def lsim(ctx, A, B, C, D, U, t, x0=None, interp="zoh", return_states=True):
    """Fixed-step simulation of dx/dt = A x + B u, y = C x + D u on the time grid t
    (1-D, evenly spaced; its first point is x0's time).  U [T, m] or [batch, T, m];
    x0 [n] or [batch, n].  interp: "zoh" (input held over each step) or "foh" (linear
    between samples).  Returns (y, x) shaped like U with m replaced by p and n (x None
    when return_states is False)."""
    from . import pararnn_lsim
    single = U.dim() == 2
    U3 = U.unsqueeze(0) if single else U
    if U3.dim() != 3:
        raise ValueError("U must be [T, m] or [batch, T, m]")
    batch, T, m = U3.shape
    n, p = A.shape[0], C.shape[0]
    # the C ABI takes bare pointers: every operand's shape is checked here
    if A.shape != (n, n) or B.shape != (n, m) or C.shape != (p, n) or (D is not None and D.shape != (p, m)):
        raise ValueError(f"shapes: A {tuple(A.shape)}, B {tuple(B.shape)}, C {tuple(C.shape)}, "
                         f"D {None if D is None else tuple(D.shape)} do not fit n = {n}, m = {m}, p = {p}")
    if x0 is not None and x0.shape not in ((n,), (batch, n)):
        raise ValueError(f"x0 must be [{n}] or [{batch}, {n}]")
    tt = torch.as_tensor(t, dtype=torch.float64).cpu().reshape(-1)
    if tt.numel() != T:
        raise ValueError("t must have one point per input sample")
    dt = float(tt[1] - tt[0]) if T > 1 else 1.0
    if T > 2 and float((tt.diff() - dt).abs().max()) > 1e-6 * max(abs(dt), 1e-30) + 1e-12:
        raise ValueError("lsim needs a fixed-step time grid")
    if x0 is not None:
        x0 = x0.reshape(1, n).expand(batch, n).contiguous() if x0.dim() == 1 else x0.contiguous()
    dev = U.device
    y = torch.empty(batch, T, p, device=dev, dtype=torch.float32)
    x = torch.empty(batch, T, n, device=dev, dtype=torch.float32) if return_states else None
    pararnn_lsim(ctx, A.contiguous(), B.contiguous(), C.contiguous(), None if D is None else D.contiguous(),
                 U3.contiguous(), x0, dt, {"zoh": 0, "foh": 1}[interp], y, x)
    if single:
        return y[0], (None if x is None else x[0])
    return y, x


def linear_scan(ctx, kind, J, b, h0=None, reverse=False):
    from . import PARARNN_SCAN_BLOCK2, PARARNN_SCAN_DENSE, PARARNN_SCAN_DIAG
    k = {"diag": PARARNN_SCAN_DIAG, "block2": PARARNN_SCAN_BLOCK2, "dense": PARARNN_SCAN_DENSE}[kind]
    B, T, N = b.shape[:3]
    S = 2 if kind == "block2" else 1
    _need(b, B * T * N * S, "b")
    _need(J, B * T * N * (N if kind == "dense" else S * S), "J")
    _need(h0, B * N * S, "h0")
    out = torch.empty_like(b)
    pararnn_linear_scan(ctx, k, J, b, h0, out, B, T, N, reverse)
    return out


def linear_scan_noalloc(kind, J, b, h0=None, reverse=False, status_out=None, h_out=None, stream=None):
    """The allocation-free scan (diag or block2) on the current device and stream.

    Checks every operand's element count before the pointer-only C call.  Returns
    (h_out, status_out); status_out (one int32 on the device) is non-zero after the
    call when a bounded wait ran out."""
    from . import PARARNN_SCAN_BLOCK2, PARARNN_SCAN_DIAG, pararnn_linear_scan_noalloc
    k = {"diag": PARARNN_SCAN_DIAG, "block2": PARARNN_SCAN_BLOCK2}[kind]
    B, T, N = b.shape[:3]
    S = 2 if kind == "block2" else 1
    _need(b, B * T * N * S, "b")
    _need(J, B * T * N * S * S, "J")
    _need(h0, B * N * S, "h0")
    _need(h_out, B * T * N * S, "h_out")
    _need(status_out, 1, "status_out")
    if h_out is None:
        h_out = torch.empty_like(b)
    if status_out is None:
        status_out = torch.zeros(1, device=b.device, dtype=torch.int32)
    pararnn_linear_scan_noalloc(k, J, b, h0, h_out, B, T, N, reverse, status_out=status_out, stream=stream)
    return h_out, status_out


def adjoint_backward(ctx, cell, B, T, H, *, xproj, a, peep=None, h0=None, h, grad_h):
    """Adjoint gradients at states h.  Returns (grad_xproj, grad_params, grad_h0)."""
    dev = xproj.device
    S = 2 if cell in ("lstm", "lstm_quasi") else 1
    _need(xproj, B * T * 3 * H, "xproj [B, T, 3, H]")
    _need(a, 3 * H, "a [3, H]")
    _need(peep, 2 * H, "peep [2, H]")
    _need(h0, B * H * S, "h0")
    _need(h, B * T * H * S, "h")
    _need(grad_h, B * T * H * S, "grad_h")
    prm = make_params(CELLS[cell], B, T, H, 0, a=a, peep=peep)
    gx = torch.empty(B, T, 3, H, device=dev, dtype=torch.float32)
    lstm = cell in ("lstm", "lstm_quasi")
    gp = torch.empty(5 if lstm else 3, H, device=dev, dtype=torch.float32)
    gh0 = torch.empty((B, H, 2) if lstm else (B, H), device=dev, dtype=torch.float32)
    pararnn_adjoint_backward(ctx, xproj, prm, h0, h, grad_h, gx, gp, gh0)
    return gx, gp, gh0


def layer_backward(ctx, cell, B, T, H, *, xproj, a, peep=None, h0=None, h, grad_h, x, W):
    """Backward pass of a layer with bf16 x [B, T, K] and W [3H, K]: the adjoint at states h
    and the projection's reverse pass, grad_xproj handed over in bf16.  Returns
    (grad_x, grad_W, grad_bias, grad_params, grad_h0)."""
    from . import pararnn_layer_backward
    dev = xproj.device
    S = 2 if cell in ("lstm", "lstm_quasi") else 1
    K = x.shape[-1]
    _need(xproj, B * T * 3 * H, "xproj [B, T, 3, H]")
    _need(a, 3 * H, "a [3, H]")
    _need(peep, 2 * H, "peep [2, H]")
    _need(h0, B * H * S, "h0")
    _need(h, B * T * H * S, "h")
    _need(grad_h, B * T * H * S, "grad_h")
    _need(x, B * T * K, "x [B, T, K]")
    _need(W, 3 * H * K, "W [3H, K]")
    prm = make_params(CELLS[cell], B, T, H, 0, a=a, peep=peep)
    lstm = cell in ("lstm", "lstm_quasi")
    gxi = torch.empty(B, T, K, device=dev, dtype=torch.float32)
    gW = torch.empty(3 * H, K, device=dev, dtype=torch.float32)
    gb = torch.empty(3 * H, device=dev, dtype=torch.float32)
    gp = torch.empty(5 if lstm else 3, H, device=dev, dtype=torch.float32)
    gh0 = torch.empty((B, H, 2) if lstm else (B, H), device=dev, dtype=torch.float32)
    pararnn_layer_backward(ctx, xproj, prm, h0, h, grad_h, x, W, gxi, gW, gb, gp, gh0)
    return gxi, gW, gb, gp, gh0
