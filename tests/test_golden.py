"""The oracle against its stored outputs (tests/golden/oracle_workloads.json, written by
tests/golden/make_golden.py from the oracle alone).  Any later change to the oracle's
arithmetic shows up here; the GPU tests compare the CUDA path to the same records.
Only the cheap workloads are recomputed on CPU."""
import json
import os

import numpy as np
import pytest

import oracle
from nonlinear_rnn_solve_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "oracle_workloads.json")


def test_golden_covers_every_workload():
    rec = json.load(open(GOLDEN))
    assert set(rec) == set(wl.WORKLOADS)
    for name, r in rec.items():
        assert r["iters"] == len(r["deltas"]) and r["iters"] >= 1


@pytest.mark.parametrize("name", ["gru_b1_t1024_in4_h8", "gru_b16_t1048576_in2_h1",
                                  "tanh_b16_t65536_in4_n8_quasi"])
def test_oracle_reproduces_golden(name):
    r = json.load(open(GOLDEN))[name]
    w = wl.WORKLOADS[name]
    inp = wl.generate(w, with_grad=False)
    m = oracle.model_from_inputs(w.cell, inp, quasi=w.quasi)
    _, iters, d = m.newton(inp["h0"], max_iters=r["cap_used"], tol=w.tol)
    assert iters == r["iters"]
    np.testing.assert_allclose(d, np.array(r["deltas"], dtype=float), rtol=1e-9, atol=1e-15)
