"""GPU parity of the least-squares scale refit (nq_ls_refit) against the FP64 oracle.

From the scales nq_lbadmm extracted, both sides run the same number of alternating
sweeps with the packed signs fixed; the refitted s1, s2 agree within 1e-4 relative to
their largest entry (FP32 sums inside a tile, FP64 across tiles), the reported error
within 1e-5 of the oracle's, and it is never above the error before the refit.
"""
import numpy as np
import pytest
import torch

from conftest import max_rel
from oracle import lbadmm as O
from oracle import refit as R

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("m,n,r,dtype,precond", [(512, 384, 64, torch.float32, False),
                                                 (700, 900, 100, torch.bfloat16, True),
                                                 (257, 129, 33, torch.float32, True),
                                                 (2048, 1024, 500, torch.bfloat16, False)])
def test_refit_matches_oracle(nq, m, n, r, dtype, precond):
    g = torch.Generator().manual_seed(m + n + r)
    W = (torch.randn(m, n, generator=g) * 0.02).to(dtype)
    d_in = d_out = None
    if precond:
        d_in = torch.exp(0.5 * torch.randn(n, generator=g)).cuda()
        d_out = torch.exp(0.5 * torch.randn(m, generator=g)).cuda()
    res = nq.nq_lbadmm(W.cuda(), r, d_in, d_out, iters=8)
    e0 = res["rel_err"]
    s1, s2 = res["s1"].clone(), res["s2"].clone()
    Us = O.unpack_signs(res["U_packed"].cpu().numpy().view(np.uint32), r)
    Vs = O.unpack_signs(res["V_packed"].cpu().numpy().view(np.uint32), r)
    Wt = W.double().numpy()
    if precond:
        Wt = d_out.cpu().double().numpy()[:, None] * Wt * d_in.cpu().double().numpy()[None, :]
    r1, r2, errors = R.ls_refit(Wt, Us, Vs, s1.cpu().double().numpy(), s2.cpu().double().numpy(),
                                sweeps=3)
    e = nq.nq_ls_refit(W.cuda(), res["U_packed"], res["V_packed"], r, s1, s2, d_in, d_out,
                       sweeps=3)
    assert max_rel(s1.cpu().numpy(), r1) <= 1e-4
    assert max_rel(s2.cpu().numpy(), r2) <= 1e-4
    assert abs(e - errors[-1]) <= 1e-5 * errors[-1], (e, errors)
    assert abs(errors[0] - e0) <= 1e-5 * e0          # the oracle starts from the same error
    assert e <= e0 * (1 + 1e-6)


def test_refit_of_planted_scales_is_exact(nq):
    # W~ = diag(a) P diag(b) exactly: the refit from perturbed scales drives the error to 0
    from oracle.splitmix import sign_matrix
    m, n, r = 300, 200, 20
    rng = np.random.default_rng(0)
    Us, Vs = sign_matrix(1, m, r), sign_matrix(2, n, r)
    a, b = np.exp(0.5 * rng.standard_normal(m)), np.exp(0.5 * rng.standard_normal(n))
    W = torch.from_numpy(((a[:, None] * (Us @ Vs.T)) * b[None, :]).astype(np.float32)).cuda()
    Up = torch.from_numpy(O.pack_signs(Us).view(np.int32)).cuda()
    Vp = torch.from_numpy(O.pack_signs(Vs).view(np.int32)).cuda()
    s1 = torch.from_numpy((a * np.exp(0.1 * rng.standard_normal(m))).astype(np.float32)).cuda()
    s2 = torch.from_numpy((b * np.exp(0.1 * rng.standard_normal(n))).astype(np.float32)).cuda()
    e = nq.nq_ls_refit(W, Up, Vp, r, s1, s2, sweeps=60)
    assert e < 1e-5
