"""Helpers for the GPU parity tests (test infrastructure)."""
import numpy as np
import pytest
import torch

DEV = torch.device("cuda:0")


def gpu(a, dtype=torch.float32):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV, dtype)


def host(t):
    return t.detach().cpu().numpy().astype(np.float64)


def need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def max_abs(a, b):
    return float(np.max(np.abs(np.asarray(a, np.float64) - np.asarray(b, np.float64)))) if np.size(a) else 0.0
