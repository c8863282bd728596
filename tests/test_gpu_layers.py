"""GPU parity, full size: a whole layer through the C ABI against the fp64 oracle.

input projection (tcgen05 bf16 GEMM) -> Newton forward -> residual -> adjoint backward,
for the ParaGRU layer (B 8, T 4096, H = in = 2048, bf16 inputs, 3 iterations) and the
ParaLSTM layer (B 4, T 8192, H = in = 1024, bf16 inputs, tol 1e-5).  Both sides read
the same seeded bf16 values; the oracle projects in fp64.  Bars (bf16-input path):
states within 2e-2, identical iteration counts; grad_xproj and grad_h0 within 2e-2
(scaled by their largest magnitude when it exceeds 1); grad_params, a sum over all
B*T steps whose magnitude grows with it, within 1e-3 of its largest magnitude.  The
errors reached are printed (pytest -s) and carried in every assertion message.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import host, need_gpu

from nonlinear_rnn_solve_b200 import Context, solve
from nonlinear_rnn_solve_b200 import workloads as wl

pytestmark = pytest.mark.gpu
TOL_BF16 = 2e-2


@pytest.fixture(scope="module")
def ctx():
    need_gpu()
    c = Context(0)
    yield c
    c.close()


def _bf16(a):
    return torch.from_numpy(wl.bf16_bits(a).view(np.int16)).cuda().view(torch.bfloat16)


@pytest.mark.parametrize("name", ["gru_b8_t4096_h2048_bf16", "lstm_b4_t8192_h1024_bf16"])
def test_layer_forward_backward_full_size(ctx, name):
    w = wl.WORKLOADS[name]
    inp = wl.generate(w)
    B, T, H = w.B, w.T, w.H
    f32 = lambda k: torch.from_numpy(inp[k]).cuda()
    xp = solve.input_proj(ctx.ctx, _bf16(inp["x"].reshape(B * T, w.inp)), _bf16(inp["W"]), f32("bias"))
    xp = xp.view(B, T, 3, H)
    out = solve.newton_forward(ctx.ctx, w.cell, B, T, H, xproj=xp, a=f32("a"),
                               peep=f32("peep") if w.cell == "lstm" else None, h0=f32("h0"),
                               max_iters=w.max_iters, tol=w.tol, residual=w.residual)
    gx, gp, gh0 = solve.adjoint_backward(ctx.ctx, w.cell, B, T, H, xproj=xp, a=f32("a"),
                                         peep=f32("peep") if w.cell == "lstm" else None, h0=f32("h0"),
                                         h=out["h"], grad_h=f32("g"))
    torch.cuda.synchronize()
    assert ctx.status() == 0

    oracle.set_threads(0)
    m = oracle.model_from_inputs(w.cell, inp)
    h_ref, it_ref, d_ref = m.newton(inp["h0"], max_iters=min(w.max_iters, 64), tol=w.tol)
    assert int(out["iters"].item()) == it_ref, (int(out["iters"].item()), it_ref, d_ref)
    h = host(out["h"])
    errs = {"h": float(np.abs(h - h_ref).max())}
    if w.residual:
        errs["residual"] = abs(float(out["residual"].item()) - m.residual(h_ref, inp["h0"]))
    rx, rp, rh0 = m.adjoint(h_ref, inp["g"], inp["h0"])
    got = {"grad_xproj": (host(gx), rx), "grad_params": (host(gp), rp), "grad_h0": (host(gh0), rh0)}
    for k, (g_, r_) in got.items():
        errs[k] = float(np.abs(g_ - r_).max())
        errs[k + "_max_ref"] = float(np.abs(r_).max())
    print(f"\n{name}: iters {int(out['iters'].item())}; " + ", ".join(f"{k} {v:.3e}" for k, v in errs.items()))
    assert errs["h"] <= TOL_BF16, errs
    if w.residual:
        assert errs["residual"] <= TOL_BF16, errs
    for k in ("grad_xproj", "grad_h0"):
        assert errs[k] <= TOL_BF16 * max(1.0, errs[k + "_max_ref"]), errs
    assert errs["grad_params"] <= 1e-3 * errs["grad_params_max_ref"], errs
