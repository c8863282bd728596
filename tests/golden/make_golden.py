"""Write tests/golden/oracle_workloads.json: the fp64 oracle's Newton iteration counts,
per-iteration deltas and (where asked) final residuals on every named workload at its
full size.  Calls only the oracle and the seeded input generator.

    python tests/golden/make_golden.py
"""
import json
import os
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from nonlinear_rnn_solve_b200 import workloads as wl  # noqa: E402


def main():
    out = {}
    for name, w in wl.WORKLOADS.items():
        t0 = time.time()
        inp = wl.generate(w, with_grad=False)
        m = oracle.model_from_inputs(w.cell, inp, quasi=w.quasi)
        cap = min(w.max_iters, 400)
        h, iters, d = m.newton(inp["h0"], max_iters=cap, tol=w.tol)
        rec = {"iters": iters, "deltas": [float(v) if np.isfinite(v) else str(v) for v in d[:iters]],
               "tol": w.tol, "cap_used": cap}
        if w.residual:
            rec["residual"] = m.residual(h, inp["h0"])
        if np.all(np.isfinite(h)):
            rec["h_abs_max"] = float(np.abs(h).max())
        out[name] = rec
        print(name, iters, f"{time.time() - t0:.1f}s", flush=True)
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_workloads.json"), "w") as f:
        json.dump(out, f, indent=1)


if __name__ == "__main__":
    main()
