"""GPU parity: the fused layer backward (adjoint, then the projection's reverse pass, with
grad_xproj handed over in bf16) against the two separate calls and the fp64 oracle.

The separate path (adjoint_backward with fp32 grad_xproj, then input_proj_backward,
which rounds it to bf16 nearest-even for the tensor-core products) is itself pinned to
the oracle by the projection and layer tests.  The fused path forms the same fp32
grad_xproj values and rounds them the same way (the ParaGRU adjoint also stores the
transposed copy that grad_W's product reads), so grad_x and grad_W are equal bit for
bit and grad_h0 too.  grad_params and grad_bias are sums whose order depends on thread
timing (shared and global float atomics): they are held to 1e-5 of their largest
magnitude against the separate path, and grad_bias additionally to the oracle's fp64
column sums of its own grad_xproj (1e-3 of the largest magnitude: the states differ
from the oracle's by the solve's own error).  Shapes: H a multiple of 32 (the adjoint's
TMA-fed tiles write bf16 directly) and H = 40 (the fallback through an fp32 buffer);
T ragged against the tiles; one full-size GRU layer.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import host, need_gpu

from nonlinear_rnn_solve_b200 import Context, solve
from nonlinear_rnn_solve_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ctx():
    need_gpu()
    c = Context(0)
    yield c
    c.close()


def _bf16(a):
    return torch.from_numpy(wl.bf16_bits(a).view(np.int16)).cuda().view(torch.bfloat16)


def _run(ctx, w, check_oracle):
    inp = wl.generate(w, with_grad=True)
    B, T, H, K = w.B, w.T, w.H, w.inp
    f32 = lambda k: torch.from_numpy(inp[k]).cuda()
    x = _bf16(inp["x"].reshape(B * T, K))
    W = _bf16(inp["W"])
    peep = f32("peep") if w.cell == "lstm" else None
    xp = solve.input_proj(ctx.ctx, x, W, f32("bias")).view(B, T, 3, H)
    out = solve.newton_forward(ctx.ctx, w.cell, B, T, H, xproj=xp, a=f32("a"), peep=peep, h0=f32("h0"),
                               max_iters=w.max_iters, tol=w.tol)
    h = out["h"]
    gxp, gp_ref, gh0_ref = solve.adjoint_backward(ctx.ctx, w.cell, B, T, H, xproj=xp, a=f32("a"), peep=peep,
                                                  h0=f32("h0"), h=h, grad_h=f32("g"))
    gx_ref, gW_ref, gb_ref = solve.input_proj_backward(ctx.ctx, gxp.view(B * T, 3 * H), x, W)
    gx, gW, gb, gp, gh0 = solve.layer_backward(ctx.ctx, w.cell, B, T, H, xproj=xp, a=f32("a"), peep=peep,
                                               h0=f32("h0"), h=h, grad_h=f32("g"), x=x.view(B, T, K), W=W)
    torch.cuda.synchronize()
    assert ctx.status() == 0
    assert torch.equal(gx.view(B * T, K), gx_ref), float((gx.view(B * T, K) - gx_ref).abs().max())
    assert torch.equal(gW, gW_ref), float((gW - gW_ref).abs().max())
    assert torch.equal(gh0, gh0_ref)
    for got, ref in ((gp, gp_ref), (gb, gb_ref)):
        scale = float(ref.abs().max())
        assert float((got - ref).abs().max()) <= 1e-5 * max(1.0, scale), (float((got - ref).abs().max()), scale)
    if check_oracle:
        m = oracle.model_from_inputs(w.cell, inp)
        rx, _, _ = m.adjoint(host(h).astype(np.float64), inp["g"], inp["h0"])
        rb = np.asarray(rx).reshape(B * T, 3 * H).sum(axis=0)
        scale = float(np.abs(rb).max())
        err = float(np.abs(host(gb) - rb).max())
        assert err <= 1e-3 * max(1.0, scale), (err, scale)


# (cell, B, T, H, K): H % 32 == 0 takes the bf16-writing adjoint (the ParaGRU one also
# writes the transposed copy when T % 8 == 0: T = 600 yes, T = 300 no); H = 40 the fallback
CASES = [("gru", 2, 600, 64, 72), ("gru", 2, 300, 32, 8), ("lstm", 2, 520, 64, 64), ("gru", 1, 264, 40, 16),
         ("lstm", 3, 200, 32, 24)]


@pytest.mark.parametrize("cell,B,T,H,K", CASES)
def test_layer_backward_matches_separate_calls_and_oracle(ctx, cell, B, T, H, K):
    base = wl.WORKLOADS["gru_b8_t4096_h2048_bf16" if cell == "gru" else "lstm_b4_t8192_h1024_bf16"]
    w = base.resized(B=B, T=T, H=H, inp=K, seed=11 + H + K, w_var=1.0 / K, max_iters=T,
                     tol=1e-5 if cell == "lstm" else 1e-6)
    _run(ctx, w, check_oracle=True)


def test_layer_backward_full_size_gru(ctx):
    _run(ctx, wl.WORKLOADS["gru_b8_t4096_h2048_bf16"], check_oracle=False)
