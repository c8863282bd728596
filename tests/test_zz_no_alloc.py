"""The allocation-free linear scan, checked against the context-based entry point.

pararnn_linear_scan_noalloc serves callers that cannot call cudaMalloc (device memory
owned by another allocator, loops that must not synchronise on an allocation,
services that must not hit out-of-memory after start-up).  It keeps its scratch in a
static device array instead of a context workspace.  This file is collected last so
that a failure here does not hide the other tests; it also passes on its own in a
fresh process, where its first call resolves the array on the device.
"""
import numpy as np
import pytest
import torch

from gpu_util import gpu, host, need_gpu

import nonlinear_rnn_solve_b200 as prn
from nonlinear_rnn_solve_b200 import Context, solve

pytestmark = pytest.mark.gpu
TOL = 1e-5  # the fp32 linear-scan tolerance of the scan parity tests


def _inputs(kind, B, T, N, seed):
    rng = np.random.Generator(np.random.PCG64(seed))
    if kind == "diag":
        J, b, h0 = rng.uniform(-1, 1, (B, T, N)), rng.standard_normal((B, T, N)), rng.standard_normal((B, N))
    else:
        J, b = rng.uniform(-1, 1, (B, T, N, 2, 2)), rng.standard_normal((B, T, N, 2))
        h0 = rng.standard_normal((B, N, 2))
    return gpu(J), gpu(b), gpu(h0)


@pytest.mark.parametrize("kind", ["diag", "block2"])
@pytest.mark.parametrize("shape", [(3, 5000, 40), (2, 9000, 1), (1, 1, 1)])
@pytest.mark.parametrize("reverse", [False, True])
def test_noalloc_scan_matches_context_scan_twice(kind, shape, reverse):
    need_gpu()
    B, T, N = shape
    status = torch.full((1,), 7, dtype=torch.int32, device="cuda")
    for call in range(2):  # two calls in a row: the shared scratch is reused
        J, b, h0 = _inputs(kind, B, T, N, seed=1000 * call + B * 7 + T + N)
        with Context(0) as ctx:
            ref = solve.linear_scan(ctx.ctx, kind, J, b, h0, reverse=reverse)
            torch.cuda.synchronize()
            assert ctx.status() == 0
        out = torch.full_like(b, float("nan"))
        solve.linear_scan_noalloc(kind, J, b, h0, reverse=reverse, status_out=status, h_out=out)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert float(np.max(np.abs(host(out) - host(ref)))) <= TOL


def test_noalloc_rejects_problems_beyond_the_scratch():
    need_gpu()
    B, T, N = 64, 65536, 2048  # about 1.2 GB of scratch as a diag scan: far beyond 16 MiB
    J = torch.empty(16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    # the raw mirror on purpose: the call returns before enqueuing anything
    with pytest.raises(prn.PararnnError) as e:
        prn.pararnn_linear_scan_noalloc(prn.PARARNN_SCAN_DIAG, J, J, None, J, B, T, N, status_out=status)
    assert e.value.code == prn.PARARNN_ESCRATCH


def test_noalloc_requires_a_status_word():
    need_gpu()
    J = torch.zeros(4, device="cuda")
    with pytest.raises(prn.PararnnError) as e:
        prn.pararnn_linear_scan_noalloc(prn.PARARNN_SCAN_DIAG, J, J, None, J, 1, 4, 1)
    assert e.value.code == prn.PARARNN_EINVAL
