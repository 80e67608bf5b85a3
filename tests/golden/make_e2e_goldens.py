#!/usr/bin/env python
"""Write the oracle's end-to-end results for the parity cases to e2e_oracle.txt.

Calls only the FP64 oracle (``oracle/``) on the seeded inputs of ``synth.cases``:
calibration preconditioners from the full 262144-token BF16 streams (identity where a
case has no streams), then LB-ADMM with rho = 1, lambda = 1e-4, K = 4 for the case's
iteration count, balancing, scales, packing and the reconstruction error against W~.
The GPU tests compare the library's reconstruction error on the same inputs with the
stored value (within 1 %).

    python tests/golden/make_e2e_goldens.py [case ...]     # default: every missing case

Each finished case appends one line, so the script can be stopped and resumed.
Columns: name m n r iters rel_err objective_last gamma mean_s1 mean_s2 seconds
"""
import os
import sys
import time

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

from oracle import calib as OC  # noqa: E402
from oracle import lbadmm as O  # noqa: E402
from synth.cases import CASES  # noqa: E402

OUT = os.path.join(HERE, "e2e_oracle.txt")
HEADER = """# End-to-end results of the FP64 oracle on the seeded parity cases (synth/cases.py).
# Written by tests/golden/make_e2e_goldens.py, which calls only oracle/; no value here
# comes from the CUDA path.  rho = 1, lambda = 1e-4, K = 4, V_0 seed 0.
# columns: name m n r iters rel_err objective_last gamma mean_s1 mean_s2 seconds
"""


def done_cases():
    if not os.path.exists(OUT):
        return set()
    with open(OUT) as f:
        return {ln.split()[0] for ln in f if ln.strip() and not ln.startswith("#")}


def run_case(c):
    t0 = time.time()
    W = c.weight().double().numpy()
    if c.act_stream:
        d_in, d_out, _, _ = OC.calib_precond((x.float().numpy() for x in c.act_chunks()),
                                             (g.float().numpy() for g in c.grad_chunks()))
    else:
        d_in = d_out = None
    res = O.lbadmm(W, d_in, d_out, r=c.r, rho=1.0, lam=1e-4, iters=c.iters, K=4,
                   seed=c.admm_seed)
    dt = time.time() - t0
    return (f"{c.name} {c.m} {c.n} {c.r} {c.iters} {res.rel_err:.10e} {res.objective[-1]:.10e} "
            f"{res.gamma:.10e} {float(np.mean(res.s1)):.10e} {float(np.mean(res.s2)):.10e} "
            f"{dt:.0f}")


def main(names):
    if not os.path.exists(OUT):
        with open(OUT, "w") as f:
            f.write(HEADER)
    # cheapest first (the oracle's cost grows with m n r iters)
    todo = names or sorted((n for n in CASES if n not in done_cases()),
                           key=lambda n: CASES[n].m * CASES[n].n * CASES[n].r * CASES[n].iters)
    for name in todo:
        line = run_case(CASES[name])
        with open(OUT, "a") as f:
            f.write(line + "\n")
        print(line, flush=True)


if __name__ == "__main__":
    main(sys.argv[1:])
