"""GPU parity: input projection xproj = x W^T + bias (tcgen05 bf16 GEMM, fp32 CUDA-core GEMM).

The bf16 path consumes bf16 values exactly and accumulates in fp32, so against the
fp64 matmul of the same bf16 values the error is fp32 accumulation only; the bar is
the bf16-input tolerance 2e-2 (max abs), and a tighter relative check catches any
layout or descriptor slip, which would give O(1) errors.
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


def _bf16_tensor(a):
    return torch.from_numpy(wl.bf16_bits(a).view(np.int16)).cuda().view(torch.bfloat16)


def _draw(M, K, N, seed):
    rng = np.random.default_rng(seed)
    x = wl.round_bf16(rng.standard_normal((M, K)).astype(np.float32))
    W = wl.round_bf16((rng.standard_normal((N, K)) / np.sqrt(K)).astype(np.float32))
    bias = rng.standard_normal(N).astype(np.float32)
    return x, W, bias


@pytest.mark.parametrize("MKN", [(128, 64, 256), (300, 128, 500), (1, 8, 1), (129, 72, 257), (1000, 1024, 768),
                                 (256, 2048, 6144)])
def test_bf16_projection_matches_oracle(ctx, MKN):
    M, K, N = MKN
    x, W, bias = _draw(M, K, N, seed=M + K + N)
    y = solve.input_proj(ctx.ctx, _bf16_tensor(x), _bf16_tensor(W), torch.from_numpy(bias).cuda())
    torch.cuda.synchronize()
    assert ctx.status() == 0
    ref = oracle.input_proj(x, W, bias)
    err = np.abs(host(y) - ref).max()
    assert err <= 2e-2
    assert err <= 1e-4 * max(1.0, np.abs(ref).max())


def test_bf16_projection_full_size_sampled_rows(ctx):
    """The 8 x 4096 x 2048 -> 3 x 2048 projection of the ParaGRU layer workload."""
    w = wl.WORKLOADS["gru_b8_t4096_h2048_bf16"]
    inp = wl.generate(w, with_grad=False)
    M, K, N = w.B * w.T, w.inp, 3 * w.H
    x = inp["x"].reshape(M, K)
    y = solve.input_proj(ctx.ctx, _bf16_tensor(x), _bf16_tensor(inp["W"]), torch.from_numpy(inp["bias"]).cuda())
    torch.cuda.synchronize()
    assert ctx.status() == 0
    rows = np.random.default_rng(0).choice(M, size=96, replace=False)
    rows = np.concatenate([rows, [0, M - 1, 127, 128]])
    ref = oracle.input_proj(x[rows], inp["W"], inp["bias"])
    got = host(y[torch.from_numpy(rows).cuda()])
    assert np.abs(got - ref).max() <= 2e-2
    assert np.abs(got - ref).max() <= 1e-4 * max(1.0, np.abs(ref).max())


@pytest.mark.parametrize("MKN", [(64, 16, 64), (300, 37, 500), (1, 1, 1)])
def test_f32_projection_matches_oracle(ctx, MKN):
    M, K, N = MKN
    rng = np.random.default_rng(M * K)
    x = rng.standard_normal((M, K)).astype(np.float32)
    W = rng.standard_normal((N, K)).astype(np.float32)
    bias = rng.standard_normal(N).astype(np.float32)
    y = solve.input_proj(ctx.ctx, torch.from_numpy(x).cuda(), torch.from_numpy(W).cuda(), torch.from_numpy(bias).cuda())
    torch.cuda.synchronize()
    ref = oracle.input_proj(x, W, bias)
    assert np.abs(host(y) - ref).max() <= 1e-4 * max(1.0, np.abs(ref).max())
