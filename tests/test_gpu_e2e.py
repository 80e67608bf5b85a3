"""End-to-end parity of the whole path on every benchmark configuration.

For each seeded case of ``synth.cases`` (config 2's q_proj, the 11008 x 4096 r = 1000
target layer, config 3's q/gate/down layers, config 4's k_proj, config 5's rank sweep)
the library runs calibration (full 262144-token BF16 streams) and LB-ADMM for the case's
iteration count, and its reconstruction error must lie within 1 % of the FP64 oracle's
on the same inputs.  The oracle's values are stored in tests/golden/e2e_oracle.txt by
tests/golden/make_e2e_goldens.py, which calls only the oracle.
"""
import numpy as np
import pytest
import torch

from conftest import read_golden
from synth.cases import CASES

pytestmark = pytest.mark.gpu
TOL_E2E = 0.01

GOLDEN = {row[0]: dict(m=int(row[1]), n=int(row[2]), r=int(row[3]), iters=int(row[4]),
                       rel_err=float(row[5]), objective_last=float(row[6]), gamma=float(row[7]))
          for row in read_golden("e2e_oracle.txt")}


def _inputs(case):
    W = case.weight().cuda()
    if not case.act_stream:
        return W, None, None
    acts = torch.empty(case.T, case.n, dtype=torch.bfloat16, device="cuda")
    grads = torch.empty(case.T, case.m, dtype=torch.bfloat16, device="cuda")
    for dst, chunks in ((acts, case.act_chunks()), (grads, case.grad_chunks())):
        t = 0
        for x in chunks:
            dst[t:t + x.shape[0]].copy_(x)
            t += x.shape[0]
    return W, acts, grads


@pytest.mark.parametrize("name", sorted(CASES))
def test_case_within_one_percent_of_oracle(nq, name):
    case, gold = CASES[name], GOLDEN[name]
    assert (gold["m"], gold["n"], gold["r"], gold["iters"]) == (case.m, case.n, case.r, case.iters)
    W, acts, grads = _inputs(case)
    d_in = d_out = None
    if acts is not None:
        d_in, d_out, _, _ = nq.nq_calib_precond(acts, grads)
        del acts, grads
    st = nq.LBState(case.m, case.n, case.r)
    gamma = st.prepare(W, d_in, d_out, seed=case.admm_seed)
    assert abs(gamma - gold["gamma"]) <= 1e-5 * gold["gamma"]
    obj = st.iterate(case.iters)
    res = st.finish(W, d_in, d_out)
    e = res["rel_err"]
    assert abs(e - gold["rel_err"]) <= TOL_E2E * gold["rel_err"], (e, gold["rel_err"])
    assert np.isfinite(obj).all()
    # the dedicated entry point reproduces the same error from the packed result
    e2 = nq.nq_recon_error(W, res["U_packed"], res["V_packed"], case.r, res["s1"], res["s2"],
                           d_in, d_out)
    assert abs(e2 - e) <= 1e-5 * e
