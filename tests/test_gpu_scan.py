"""GPU parity: standalone linear scans (diag, 2x2 block) against the fp64 oracle.

Tolerance: max abs error <= 1e-5 for the fp32 linear scan.  Inputs: J ~ U(-1, 1),
b ~ N(0, 1) (seeded), shapes spanning several tiles and a ragged tail, T = 1,
N not a multiple of the channel tile; N a multiple of 32 (the shared-memory staged
kernel) with T ragged against its 128- and 64-step tiles and below one tile.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import gpu, host, max_abs, need_gpu

from nonlinear_rnn_solve_b200 import Context, solve

pytestmark = pytest.mark.gpu
TOL = 1e-5


@pytest.fixture(scope="module")
def ctx():
    need_gpu()
    c = Context(0)
    yield c
    c.close()


def _draw(kind, B, T, N, seed, with_h0):
    rng = np.random.Generator(np.random.PCG64(seed))
    if kind == "diag":
        J = rng.uniform(-1, 1, (B, T, N)); b = rng.standard_normal((B, T, N)); hs = (B, N)
    else:
        J = rng.uniform(-1, 1, (B, T, N, 2, 2)); b = rng.standard_normal((B, T, N, 2)); hs = (B, N, 2)
    h0 = rng.standard_normal(hs) if with_h0 else None
    f = lambda a: None if a is None else a.astype(np.float32)
    return f(J), f(b), f(h0)


SHAPES = [(1, 1, 1), (2, 5, 3), (3, 4097, 1), (2, 8193, 1), (2, 300, 33), (1, 1000, 8), (4, 1025, 2),
          (2, 129, 64), (1, 3000, 17), (2, 1000, 32), (1, 5000, 96), (3, 70, 32)]


@pytest.mark.parametrize("kind", ["diag", "block2"])
@pytest.mark.parametrize("reverse", [False, True])
@pytest.mark.parametrize("shape", SHAPES)
def test_scan_matches_oracle(ctx, kind, reverse, shape):
    B, T, N = shape
    J, b, h0 = _draw(kind, B, T, N, seed=B * 1000003 + T * 31 + N, with_h0=(T % 2 == 1))
    out = solve.linear_scan(ctx.ctx, kind, gpu(J), gpu(b), None if h0 is None else gpu(h0), reverse=reverse)
    torch.cuda.synchronize()
    assert ctx.status() == 0
    ref = oracle.linear_scan(kind, J, b, h0, reverse=reverse)
    assert max_abs(host(out), ref) <= TOL


# N = 20, 44: rows of a multiple of 4 floats copied in 16-byte pieces into the 32- and
# 64-wide padded tiles, whose padding stays zero; N = 13: the element-wise staging
@pytest.mark.parametrize("N", [1, 5, 8, 13, 20, 32, 44, 64])
@pytest.mark.parametrize("reverse", [False, True])
@pytest.mark.parametrize("BT", [(2, 300), (1, 1), (3, 1025)])
def test_dense_scan_matches_oracle(ctx, N, reverse, BT):
    B, T = BT
    rng = np.random.Generator(np.random.PCG64(N * 1000 + T))
    a = 0.9 * np.sqrt(3.0 / N)  # spectral radius near 0.9
    J = rng.uniform(-a, a, (B, T, N, N)).astype(np.float32)
    b = rng.standard_normal((B, T, N)).astype(np.float32)
    h0 = rng.standard_normal((B, N)).astype(np.float32) if T % 2 else None
    out = solve.linear_scan(ctx.ctx, "dense", gpu(J), gpu(b), None if h0 is None else gpu(h0), reverse=reverse)
    torch.cuda.synchronize()
    assert ctx.status() == 0
    assert max_abs(host(out), oracle.linear_scan("dense", J, b, h0, reverse=reverse)) <= TOL


def test_scan_long_sequence_many_tiles(ctx):
    """16 sequences of 2^20 steps at N = 1: 4096 tiles, full decoupled look-back."""
    B, T, N = 16, 1 << 20, 1
    J, b, h0 = _draw("diag", B, T, N, seed=7, with_h0=True)
    out = solve.linear_scan(ctx.ctx, "diag", gpu(J), gpu(b), gpu(h0))
    torch.cuda.synchronize()
    assert ctx.status() == 0
    assert max_abs(host(out), oracle.linear_scan("diag", J, b, h0)) <= TOL
