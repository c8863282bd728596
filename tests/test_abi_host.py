"""Host-side checks of the C ABI (no GPU needed, no compute calls).

The library must load, export every entry point include/pararnn.h declares, and
reject bad arguments with status codes before touching the device.
"""
import ctypes
import os
import re
import subprocess

import pytest

import nonlinear_rnn_solve_b200 as prn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pararnn.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(pararnn_[a-z_0-9]+)\s*\(", src)))


def test_library_builds_and_loads():
    from nonlinear_rnn_solve_b200 import build
    path = build.build()
    assert os.path.exists(path)
    assert prn.lib() is not None


def test_every_declared_symbol_is_exported():
    names = declared_functions()
    assert len(names) >= 10
    L = prn.lib()
    missing = [n for n in names if not hasattr(L, n)]
    assert not missing, missing
    out = subprocess.run(["nm", "-D", "--defined-only", prn.LIB_PATH], capture_output=True, text=True).stdout
    for n in names:
        assert re.search(rf"\bT {n}$", out, flags=re.M), n
    assert sorted(prn.EXPORTED) == names


def test_strerror_covers_codes():
    for code in [0, 1, -1, -2, -3, -4, -5, -6, -7]:
        assert prn.strerror(code) != "unknown status"
    assert prn.strerror(12345) == "unknown status"


def test_null_context_and_pointers_are_rejected():
    L = prn.lib()
    EINVAL = prn.PARARNN_EINVAL
    p = prn.pararnn_params()
    assert L.pararnn_create(None, 0, None) == EINVAL
    assert L.pararnn_destroy(None) == EINVAL
    assert L.pararnn_set_stream(None, None) == EINVAL
    assert L.pararnn_newton_forward(None, None, ctypes.byref(p), None, None, 1, 1e-6, None, None, None) == EINVAL
    assert L.pararnn_linear_scan(None, 0, None, None, None, None, 1, 1, 1, 0) == EINVAL
    assert L.pararnn_adjoint_backward(None, None, ctypes.byref(p), None, None, None, None, None, None) == EINVAL
    assert L.pararnn_input_proj(None, None, 0, None, None, None, 1, 1, 1) == EINVAL
    assert L.pararnn_input_proj_backward(None, None, None, 0, None, None, None, None, 1, 1, 1) == EINVAL
    assert L.pararnn_lsim(None, None, None, None, None, 1, 1, 1, None, None, 0.1, 0, 1, 1, None, None) == EINVAL
    assert L.pararnn_layer_backward(None, None, ctypes.byref(p), None, None, None, None, None, 8, None, None, None,
                                    None, None) == EINVAL
    st = ctypes.c_int()
    assert L.pararnn_get_status(None, ctypes.byref(st)) == EINVAL
    assert L.pararnn_debug_set(None, 1, 5) == EINVAL
    assert L.pararnn_last_launch_count(None) == 0


@pytest.mark.skipif(os.path.exists("/dev/nvidia0"), reason="a GPU is present")
def test_create_without_gpu_fails_cleanly():
    ctx = ctypes.c_void_p()
    rc = prn.lib().pararnn_create(ctypes.byref(ctx), 0, None)
    assert rc < 0 and not ctx.value


def test_binding_refuses_cpu_tensors():
    import torch
    with pytest.raises(TypeError):
        prn._p(torch.zeros(4))


def test_lsim_binding_checks_the_time_grid_on_the_host():
    """The fixed-step grid and its length are checked before any device call."""
    import numpy as np
    import torch
    from nonlinear_rnn_solve_b200 import solve
    A, B, C = torch.zeros(2, 2), torch.zeros(2, 1), torch.zeros(1, 2)
    U = torch.zeros(6, 1)
    with pytest.raises(ValueError):  # uneven steps
        solve.lsim(None, A, B, C, None, U, np.array([0.0, 1.0, 2.0, 3.5, 4.0, 5.0]))
    with pytest.raises(ValueError):  # one time per sample
        solve.lsim(None, A, B, C, None, U, np.arange(5) * 0.1)
    with pytest.raises(TypeError):  # even grid: reaches the binding, which takes CUDA tensors only
        solve.lsim(None, A, B, C, None, U, np.arange(6) * 0.1)
    t = np.arange(6) * 0.1
    with pytest.raises(ValueError):  # B with 2 inputs, U with 1
        solve.lsim(None, A, torch.zeros(2, 2), C, None, U, t)
    with pytest.raises(ValueError):  # C not [p, n]
        solve.lsim(None, A, B, torch.zeros(1, 3), None, U, t)
    with pytest.raises(ValueError):  # D not [p, m]
        solve.lsim(None, A, B, C, torch.zeros(2, 1), U, t)
    with pytest.raises(ValueError):  # x0 not [n]
        solve.lsim(None, A, B, C, None, U, t, x0=torch.zeros(3))


def test_wrappers_check_operand_sizes_before_the_pointer_only_calls():
    """A wrong-sized operand raises ValueError on the host (the C calls take bare
    pointers and would read or write past it)."""
    import torch
    from nonlinear_rnn_solve_b200 import solve
    z = torch.zeros
    with pytest.raises(ValueError):  # block2 J must be [B, T, N, 2, 2]
        solve.linear_scan(None, "block2", z(2, 5, 3), z(2, 5, 3, 2))
    with pytest.raises(ValueError):  # h0 [B, N]
        solve.linear_scan(None, "diag", z(2, 5, 3), z(2, 5, 3), z(3))
    with pytest.raises(ValueError):  # xproj [B, T, 3, H]
        solve.newton_forward(None, "gru", 2, 5, 4, xproj=z(2, 5, 4), a=z(3, 4))
    with pytest.raises(ValueError):  # LSTM h0 holds (c, h) pairs
        solve.newton_forward(None, "lstm", 2, 5, 4, xproj=z(2, 5, 3, 4), a=z(3, 4), peep=z(2, 4), h0=z(2, 4))
    with pytest.raises(ValueError):  # tanh A [n, n]
        solve.newton_forward(None, "tanh", 2, 5, 4, xproj=z(2, 5, 4), A=z(4, 3))
    with pytest.raises(ValueError):  # grad_h like h
        solve.adjoint_backward(None, "gru", 2, 5, 4, xproj=z(2, 5, 3, 4), a=z(3, 4), h=z(2, 5, 4), grad_h=z(2, 4, 4))
    with pytest.raises(ValueError):  # W [N, K]
        solve.input_proj(None, z(6, 8), z(16, 7))
    with pytest.raises(ValueError):  # grad_xproj [M, N]
        solve.input_proj_backward(None, z(6, 15), z(6, 8), z(16, 8))
    with pytest.raises(ValueError):  # layer backward: x [B, T, K]
        solve.layer_backward(None, "gru", 2, 8, 32, xproj=z(2, 8, 3, 32), a=z(3, 32), h=z(2, 8, 32),
                             grad_h=z(2, 8, 32), x=z(2, 7, 16), W=z(96, 16))
    with pytest.raises(ValueError):  # layer backward: W [3H, K]
        solve.layer_backward(None, "lstm", 2, 8, 32, xproj=z(2, 8, 3, 32), a=z(3, 32), peep=z(2, 32),
                             h=z(2, 8, 32, 2), grad_h=z(2, 8, 32, 2), x=z(2, 8, 16), W=z(64, 16))
    with pytest.raises(ValueError):  # allocation-free scan: block2 J [B, T, N, 2, 2]
        solve.linear_scan_noalloc("block2", z(2, 5, 3, 2), z(2, 5, 3, 2))
    with pytest.raises(ValueError):  # allocation-free scan: h_out like b
        solve.linear_scan_noalloc("diag", z(2, 5, 3), z(2, 5, 3), h_out=z(2, 5, 2))
    with pytest.raises(ValueError):  # allocation-free scan: one status word
        solve.linear_scan_noalloc("diag", z(2, 5, 3), z(2, 5, 3), status_out=z(2, dtype=torch.int32))


def test_noalloc_scan_rejects_a_missing_status_word_on_the_host():
    """A NULL status word is refused before any device call (a timeout would otherwise go
    unreported)."""
    L = prn.lib()
    x = ctypes.c_void_p(256)
    assert L.pararnn_linear_scan_noalloc(0, x, x, None, x, 1, 4, 1, 0, None, None) == prn.PARARNN_EINVAL
