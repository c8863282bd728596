"""Newton (DEER) / quasi-Newton evaluation of nonlinear RNNs on B200 (sm_100a).

Thin Python binding of the C ABI in ``include/pararnn.h``: every function here only
marshals PyTorch CUDA tensors into pointers and sizes and calls ``libpararnn.so``,
where every step of the computation runs.  There is no CPU fallback: without the
built library the calls raise.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "_lib", "libpararnn.so")

PARARNN_OK = 0
PARARNN_NOTCONVERGED = 1
PARARNN_EINVAL = -1
PARARNN_EALIGN = -2
PARARNN_ECUDA = -3
PARARNN_ENOMEM = -4
PARARNN_ENONFINITE = -5
PARARNN_ETIMEOUT = -6
PARARNN_EUNSUPPORTED = -7
PARARNN_ESCRATCH = -8

PARARNN_GRU_DIAG = 0
PARARNN_LSTM_CIFG_PEEP = 1
PARARNN_RNN_TANH_DENSE = 2
PARARNN_RNN_TANH_QUASI = 3
PARARNN_LSTM_CIFG_PEEP_QUASI = 4
PARARNN_SOLVER_NEWTON = 0
PARARNN_SOLVER_JACOBI = 1
PARARNN_SOLVER_PICARD = 2
PARARNN_SOLVER_ELK = 3

PARARNN_SCAN_DIAG = 0
PARARNN_SCAN_BLOCK2 = 1
PARARNN_SCAN_DENSE = 2

PARARNN_F32 = 0
PARARNN_BF16 = 1

EXPORTED = [
    "pararnn_create", "pararnn_destroy", "pararnn_set_stream", "pararnn_input_proj",
    "pararnn_newton_forward", "pararnn_linear_scan", "pararnn_adjoint_backward",
    "pararnn_get_status", "pararnn_strerror", "pararnn_debug_set", "pararnn_last_launch_count",
    "pararnn_linear_scan_noalloc", "pararnn_input_proj_backward", "pararnn_lsim",
    "pararnn_layer_backward",
]


class PararnnError(RuntimeError):
    def __init__(self, code: int, what: str = ""):
        self.code = code
        super().__init__(f"{what}: {strerror(code)} ({code})")


class pararnn_params(ctypes.Structure):
    _fields_ = [("cell", ctypes.c_int), ("B", ctypes.c_int), ("T", ctypes.c_int),
                ("H", ctypes.c_int), ("in_", ctypes.c_int),
                ("a", ctypes.c_void_p), ("peep", ctypes.c_void_p), ("A", ctypes.c_void_p),
                ("x", ctypes.c_void_p), ("W", ctypes.c_void_p), ("bias", ctypes.c_void_p),
                ("solver", ctypes.c_int), ("damping", ctypes.c_float)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libpararnn.so (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m nonlinear_rnn_solve_b200.build` (no CPU fallback exists)")
        L = ctypes.CDLL(LIB_PATH)
        vp, i, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
        L.pararnn_create.argtypes = [ctypes.POINTER(vp), i, vp]
        L.pararnn_destroy.argtypes = [vp]
        L.pararnn_set_stream.argtypes = [vp, vp]
        L.pararnn_input_proj.argtypes = [vp, vp, i, vp, vp, vp, i, i, i]
        L.pararnn_newton_forward.argtypes = [vp, vp, ctypes.POINTER(pararnn_params), vp, vp, i, f,
                                             vp, vp, vp]
        L.pararnn_linear_scan.argtypes = [vp, i, vp, vp, vp, vp, i, i, i, i]
        L.pararnn_adjoint_backward.argtypes = [vp, vp, ctypes.POINTER(pararnn_params), vp, vp, vp,
                                               vp, vp, vp]
        L.pararnn_get_status.argtypes = [vp, ctypes.POINTER(i)]
        L.pararnn_strerror.argtypes = [i]
        L.pararnn_strerror.restype = ctypes.c_char_p
        L.pararnn_debug_set.argtypes = [vp, i, ctypes.c_longlong]
        L.pararnn_last_launch_count.argtypes = [vp]
        L.pararnn_linear_scan_noalloc.argtypes = [i, vp, vp, vp, vp, i, i, i, i, vp, vp]
        L.pararnn_input_proj_backward.argtypes = [vp, vp, vp, i, vp, vp, vp, vp, i, i, i]
        L.pararnn_lsim.argtypes = [vp, vp, vp, vp, vp, i, i, i, vp, vp, ctypes.c_double, i, i, i, vp, vp]
        L.pararnn_layer_backward.argtypes = [vp, vp, ctypes.POINTER(pararnn_params), vp, vp, vp, vp, vp, i,
                                             vp, vp, vp, vp, vp]
        for name in EXPORTED:
            if getattr(L, name).restype is None and name != "pararnn_strerror":
                getattr(L, name).restype = i
        _lib = L
    return _lib


def strerror(code: int) -> str:
    try:
        return lib().pararnn_strerror(int(code)).decode()
    except ImportError:
        return f"status {code}"


def _check(rc: int, what: str) -> int:
    if rc < 0:
        raise PararnnError(rc, what)
    return rc


def _p(t, dtype=None):
    """Device pointer of a contiguous CUDA tensor (or None)."""
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"expected {dtype}, got {t.dtype}")
    return ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


# ------------------------------------------------------------------ C-ABI mirrors
def pararnn_create(device: int = 0, stream=None) -> ctypes.c_void_p:
    ctx = ctypes.c_void_p()
    _check(lib().pararnn_create(ctypes.byref(ctx), int(device), _stream_handle(stream)), "pararnn_create")
    return ctx


def pararnn_destroy(ctx) -> None:
    _check(lib().pararnn_destroy(ctx), "pararnn_destroy")


def pararnn_set_stream(ctx, stream=None) -> None:
    _check(lib().pararnn_set_stream(ctx, _stream_handle(stream)), "pararnn_set_stream")


def make_params(cell, B, T, H, inp=0, a=None, peep=None, A=None, x=None, W=None, bias=None, solver=0,
                damping=0.0):
    f32 = torch.float32
    return pararnn_params(int(cell), int(B), int(T), int(H), int(inp), _p(a, f32), _p(peep, f32),
                          _p(A, f32), _p(x, f32), _p(W, f32), _p(bias, f32), int(solver), float(damping))


def pararnn_input_proj(ctx, x, W, bias, xproj) -> None:
    """xproj[M, N] = x[M, K] @ W[N, K]^T + bias (x, W both bf16 or both fp32)."""
    if x.dtype != W.dtype or x.dtype not in (torch.bfloat16, torch.float32):
        raise TypeError("x and W must both be bf16 or both fp32")
    dt = PARARNN_BF16 if x.dtype == torch.bfloat16 else PARARNN_F32
    K = x.shape[-1]
    M = x.numel() // K
    N = W.shape[0]
    _check(lib().pararnn_input_proj(ctx, _p(x), dt, _p(W), _p(bias, torch.float32),
                                    _p(xproj, torch.float32), M, K, N), "pararnn_input_proj")


def pararnn_lsim(ctx, A, Bm, C, D, U, x0, dt, interp, y_out, x_out) -> None:
    """Fixed-step linear simulation: A [n,n], Bm [n,m], C [p,n], D [p,m] or None,
    U [batch,T,m], x0 [batch,n] or None, y_out [batch,T,p], x_out [batch,T,n] or None."""
    f32 = torch.float32
    n, m = Bm.shape
    p = C.shape[0]
    batch, T = U.shape[0], U.shape[1]
    _check(lib().pararnn_lsim(ctx, _p(A, f32), _p(Bm, f32), _p(C, f32), _p(D, f32), n, m, p, _p(U, f32),
                              _p(x0, f32), float(dt), int(interp), batch, T, _p(y_out, f32), _p(x_out, f32)),
           "pararnn_lsim")


def pararnn_input_proj_backward(ctx, grad_xproj, x, W, grad_x, grad_W, grad_bias) -> None:
    """grad_x = grad_xproj @ W, grad_W = grad_xproj^T @ x, grad_bias = column sums
    (x, W both bf16 or both fp32; any output may be None)."""
    if x.dtype != W.dtype or x.dtype not in (torch.bfloat16, torch.float32):
        raise TypeError("x and W must both be bf16 or both fp32")
    dt = PARARNN_BF16 if x.dtype == torch.bfloat16 else PARARNN_F32
    K = x.shape[-1]
    M = x.numel() // K
    N = W.shape[0]
    f32 = torch.float32
    _check(lib().pararnn_input_proj_backward(ctx, _p(grad_xproj, f32), _p(x), dt, _p(W), _p(grad_x, f32),
                                             _p(grad_W, f32), _p(grad_bias, f32), M, K, N),
           "pararnn_input_proj_backward")


def pararnn_newton_forward(ctx, xproj, params, h0, h_out, max_iters, tol, iters_out,
                           final_delta_out=None, residual_out=None) -> None:
    f32 = torch.float32
    _check(lib().pararnn_newton_forward(ctx, _p(xproj, f32), ctypes.byref(params), _p(h0, f32),
                                        _p(h_out, f32), int(max_iters), float(tol),
                                        _p(iters_out, torch.int32), _p(final_delta_out, f32),
                                        _p(residual_out, f32)), "pararnn_newton_forward")


def pararnn_linear_scan(ctx, kind, J, b, h0, h_out, B, T, N, reverse=False) -> None:
    f32 = torch.float32
    _check(lib().pararnn_linear_scan(ctx, int(kind), _p(J, f32), _p(b, f32), _p(h0, f32),
                                     _p(h_out, f32), int(B), int(T), int(N), int(bool(reverse))),
           "pararnn_linear_scan")


def pararnn_adjoint_backward(ctx, xproj, params, h0, h, grad_h, grad_xproj, grad_params,
                             grad_h0=None) -> None:
    f32 = torch.float32
    _check(lib().pararnn_adjoint_backward(ctx, _p(xproj, f32), ctypes.byref(params), _p(h0, f32),
                                          _p(h, f32), _p(grad_h, f32), _p(grad_xproj, f32),
                                          _p(grad_params, f32), _p(grad_h0, f32)),
           "pararnn_adjoint_backward")


def pararnn_layer_backward(ctx, xproj, params, h0, h, grad_h, x, W, grad_x, grad_W, grad_bias,
                           grad_params, grad_h0=None) -> None:
    """Adjoint plus projection backward of a layer with bf16 x [B*T, K] and W [3H, K]
    (grad_x, grad_W, grad_bias may each be None)."""
    if x.dtype != torch.bfloat16 or W.dtype != torch.bfloat16:
        raise TypeError("x and W must both be bf16")
    f32 = torch.float32
    _check(lib().pararnn_layer_backward(ctx, _p(xproj, f32), ctypes.byref(params), _p(h0, f32), _p(h, f32),
                                        _p(grad_h, f32), _p(x), _p(W), int(x.shape[-1]), _p(grad_x, f32),
                                        _p(grad_W, f32), _p(grad_bias, f32), _p(grad_params, f32),
                                        _p(grad_h0, f32)), "pararnn_layer_backward")


def pararnn_get_status(ctx) -> int:
    st = ctypes.c_int(0)
    _check(lib().pararnn_get_status(ctx, ctypes.byref(st)), "pararnn_get_status")
    return int(st.value)


def pararnn_strerror(code: int) -> str:
    return strerror(code)


def pararnn_debug_set(ctx, knob: int, value: int) -> None:
    _check(lib().pararnn_debug_set(ctx, int(knob), int(value)), "pararnn_debug_set")


def pararnn_last_launch_count(ctx) -> int:
    return int(lib().pararnn_last_launch_count(ctx))


def pararnn_linear_scan_noalloc(kind, J, b, h0, h_out, B, T, N, reverse=False, status_out=None,
                                stream=None) -> None:
    """Allocation-free diag / block2 scan (see include/pararnn.h); current device and stream."""
    f32 = torch.float32
    _check(lib().pararnn_linear_scan_noalloc(int(kind), _p(J, f32), _p(b, f32), _p(h0, f32),
                                             _p(h_out, f32), int(B), int(T), int(N), int(bool(reverse)),
                                             _p(status_out, torch.int32), _stream_handle(stream)),
           "pararnn_linear_scan_noalloc")


# ------------------------------------------------------------------ convenience
class Context:
    """Owns a pararnn context bound to a device and stream (closes on exit)."""

    def __init__(self, device: int | None = None, stream=None):
        self.device = torch.cuda.current_device() if device is None else int(device)
        self.ctx = pararnn_create(self.device, stream)

    def close(self):
        if self.ctx is not None:
            pararnn_destroy(self.ctx)
            self.ctx = None

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def status(self) -> int:
        return pararnn_get_status(self.ctx)
