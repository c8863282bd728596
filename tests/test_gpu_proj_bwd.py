"""GPU parity: reverse pass of the input projection (grad_x, grad_W, grad_bias).

bf16 path: the products consume grad_xproj rounded to bf16 (nearest-even) and the
bf16 values of x and W exactly, with fp32 accumulation; the oracle gets the same
rounded grad_xproj, so the difference is fp32 accumulation only.  The bias gradient
sums the fp32 grad_xproj.  fp32 path: CUDA-core products of the fp32 values.  Bar:
max abs error <= 1e-4 x max(1, max |reference|) (a layout or operand slip gives O(1)
errors), inside the 2e-2 bf16-path tolerance.  Shapes: ragged against the 128 x 256
GEMM tiles and the 64 x 64 transpose tiles; the full LLM-width shapes are checked on
sampled rows and columns.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import gpu, host, need_gpu

from nonlinear_rnn_solve_b200 import Context, PararnnError, solve
from nonlinear_rnn_solve_b200 import workloads as wl

pytestmark = pytest.mark.gpu
REL = 1e-4


@pytest.fixture(scope="module")
def ctx():
    need_gpu()
    c = Context(0)
    yield c
    c.close()


def _bf16_tensor(a):
    return torch.from_numpy(wl.bf16_bits(a).view(np.int16)).cuda().view(torch.bfloat16)


def _draw(M, K, N, seed):
    rng = np.random.default_rng(seed)
    x = wl.round_bf16(rng.standard_normal((M, K)).astype(np.float32))
    W = wl.round_bf16((rng.standard_normal((N, K)) / np.sqrt(K)).astype(np.float32))
    g = rng.standard_normal((M, N)).astype(np.float32)
    return x, W, g


def _close(got, ref):
    scale = max(1.0, float(np.abs(ref).max()))
    return float(np.abs(host(got) - ref).max()) <= REL * scale


# (2368, 256, 256), (4160, 136, 264): grad_W has 2-3 output tiles over 37 / 65 K blocks of
# the contraction, so its product is split into 4 parts (ragged) and summed
@pytest.mark.parametrize("MKN", [(8, 8, 8), (136, 72, 264), (1000, 1024, 768), (64, 2048, 128), (264, 8, 520),
                                 (2368, 256, 256), (4160, 136, 264)])
def test_bf16_projection_backward_matches_oracle(ctx, MKN):
    M, K, N = MKN
    x, W, g = _draw(M, K, N, seed=M * 7 + K * 3 + N)
    gx, gW, gb = solve.input_proj_backward(ctx.ctx, gpu(g), _bf16_tensor(x), _bf16_tensor(W))
    torch.cuda.synchronize()
    assert ctx.status() == 0
    rx, rW, _ = oracle.input_proj_backward(wl.round_bf16(g), x, W)
    _, _, rb = oracle.input_proj_backward(g, x, W)
    assert _close(gx, rx) and _close(gW, rW) and _close(gb, rb)


@pytest.mark.parametrize("MKN", [(1, 1, 1), (37, 5, 29), (300, 64, 200)])
def test_f32_projection_backward_matches_oracle(ctx, MKN):
    M, K, N = MKN
    rng = np.random.default_rng(M + K + N)
    x = rng.standard_normal((M, K)).astype(np.float32)
    W = rng.standard_normal((N, K)).astype(np.float32)
    g = rng.standard_normal((M, N)).astype(np.float32)
    gx, gW, gb = solve.input_proj_backward(ctx.ctx, gpu(g), gpu(x), gpu(W))
    torch.cuda.synchronize()
    assert ctx.status() == 0
    rx, rW, rb = oracle.input_proj_backward(g, x, W)
    assert _close(gx, rx) and _close(gW, rW) and _close(gb, rb)


def test_outputs_may_be_skipped(ctx):
    x, W, g = _draw(136, 72, 264, seed=5)
    gx, gW, gb = solve.input_proj_backward(ctx.ctx, gpu(g), _bf16_tensor(x), _bf16_tensor(W), need_x=False,
                                           need_bias=False)
    torch.cuda.synchronize()
    assert gx is None and gb is None
    _, rW, _ = oracle.input_proj_backward(wl.round_bf16(g), x, W)
    assert _close(gW, rW)


def test_bf16_shape_not_multiple_of_8_is_rejected(ctx):
    x, W, g = _draw(12, 8, 8, seed=6)
    with pytest.raises(PararnnError):
        solve.input_proj_backward(ctx.ctx, gpu(g), _bf16_tensor(x), _bf16_tensor(W))


@pytest.mark.parametrize("name", ["gru_b8_t4096_h2048_bf16", "lstm_b4_t8192_h1024_bf16"])
def test_full_size_sampled(ctx, name):
    """The layer shapes (M = B*T, K = in, N = 3H): 64 sampled rows of grad_x and
    columns of grad_W against fp64 sums, and the whole bias gradient."""
    w = wl.WORKLOADS[name]
    inp = wl.generate(w)
    x = inp["x"].reshape(-1, w.inp)
    W = inp["W"]
    M, K, N = x.shape[0], w.inp, W.shape[0]
    rng = np.random.default_rng(11)
    g = rng.standard_normal((M, N)).astype(np.float32)
    gx, gW, gb = solve.input_proj_backward(ctx.ctx, gpu(g), _bf16_tensor(x), _bf16_tensor(W))
    torch.cuda.synchronize()
    assert ctx.status() == 0
    gr = wl.round_bf16(g).astype(np.float64)
    rows = rng.choice(M, 64, replace=False)
    cols = rng.choice(N, 64, replace=False)
    rx = gr[rows] @ W.astype(np.float64)
    rW = gr[:, cols].T @ x.astype(np.float64)
    rb = g.astype(np.float64).sum(axis=0)
    assert float(np.abs(host(gx[rows]) - rx).max()) <= REL * max(1.0, float(np.abs(rx).max()))
    assert float(np.abs(host(gW[cols]) - rW).max()) <= REL * max(1.0, float(np.abs(rW).max()))
    assert float(np.abs(host(gb) - rb).max()) <= REL * max(1.0, float(np.abs(rb).max()))
