"""GPU parity of the gradient-descent latent update (nq_set_latent_solver "gd") with the
oracle's gradient-descent update (oracle/gd.py).

Tolerances: a single half step of 8 steps on identical inputs within 2e-3 of max|X| in the
BF16 mode (as the exact path's single step) and 2e-4 in the FP32-accurate mode (each step
is a split-BF16 product of relative error ~1.5e-5; 8 of them, contracting); S, a, b the
same.  Over a run the two gradient-descent LB-ADMMs agree on the final reconstruction
error within 1 % and on every iteration's objective within 1 %.
"""
import numpy as np
import pytest
import torch

from conftest import max_rel
from oracle import gd as GD
from oracle import lbadmm as O
from synth import student_t_weight

pytestmark = pytest.mark.gpu


def bf16_exact(a):
    return torch.as_tensor(np.asarray(a), dtype=torch.float32).to(torch.bfloat16).float().numpy()


def _split(a):
    t = torch.from_numpy(np.asarray(a, dtype=np.float32))
    hi = t.to(torch.bfloat16)
    return hi, (t - hi.float()).to(torch.bfloat16)


@pytest.fixture
def gd_mode(nq):
    yield nq
    nq.nq_set_latent_solver("exact")


@pytest.mark.parametrize("prec,m,n,r", [("bf16", 1000, 777, 130), ("bf16", 700, 900, 257),
                                        ("fp32", 520, 600, 300), ("bf16", 2048, 1536, 1000)])
@pytest.mark.parametrize("side", [0, 1])
def test_gd_single_step_matches_oracle(gd_mode, prec, m, n, r, side):
    nq = gd_mode
    steps, rho, lam, K = 8, 1.0, 1e-4, 4
    rng = np.random.default_rng(7 * m + r + side)
    cast = bf16_exact if prec == "bf16" else (lambda a: np.asarray(a, dtype=np.float32))
    Wh = cast(rng.standard_normal((m, n)) * 0.1)
    U = cast(rng.standard_normal((m, r)) * 0.2).astype(np.float64)
    V = cast(rng.standard_normal((n, r)) * 0.2).astype(np.float64)
    SU = rng.standard_normal((m, r)).astype(np.float32)
    SV = rng.standard_normal((n, r)).astype(np.float32)
    aU, aV = [np.abs(rng.standard_normal(k)).astype(np.float32) / np.sqrt(k) for k in (m, n)]
    bU, bV = [np.abs(rng.standard_normal(r)).astype(np.float32) for _ in range(2)]
    st = nq.LBState(m, n, r, prec=prec)
    st.prepare(torch.zeros(m, n, device="cuda"), seed=0)
    hi, lo = _split(Wh)
    st.field("WHAT")[:, :n].copy_(hi.cuda())
    st.field("WHAT_LO")[:, :n].copy_(lo.cuda())
    for name, val in (("U", U), ("V", V), ("SU", SU), ("SV", SV)):
        st.field(name)[:, :r].copy_(torch.from_numpy(val).float().cuda())
    for name, val in (("AU", aU), ("BU", bU), ("AV", aV), ("BV", bV)):
        st.field(name).copy_(torch.from_numpy(val).float().cuda())
    st.sync_operands()
    nq.nq_set_latent_solver("gd", steps)
    st.half_step(side, rho, lam, K)
    assert st.check_device_error() == 0
    A = Wh.astype(np.float64) if side == 0 else Wh.astype(np.float64).T
    Y, X0 = (V, U) if side == 0 else (U, V)
    S0, a0, b0 = (SU, aU, bU) if side == 0 else (SV, aV, bV)
    S0 = S0.astype(np.float64)
    Z = O.sign_pm(S0) * np.outer(a0, b0)
    Lam = S0 - Z
    Xr, _, _, _ = GD.latent_update_gd(A, Y, Z, Lam, X0, rho, lam, steps)
    Sr = Xr + Lam
    _, ar, br = O.svid(Sr, K)
    tag = "U" if side == 0 else "V"
    tol = 2e-3 if prec == "bf16" else 2e-4
    X = st.field(tag)[:, :r].cpu().double().numpy()
    S = st.field("S" + tag)[:, :r].cpu().double().numpy()
    assert max_rel(X, Xr) <= tol
    assert max_rel(S, Sr) <= tol
    assert max_rel(st.field("A" + tag).cpu().double().numpy(), ar) <= tol
    assert max_rel(st.field("B" + tag).cpu().double().numpy(), br) <= tol


def test_gd_run_matches_oracle(gd_mode):
    nq = gd_mode
    m, n, r, iters, steps = 1024, 768, 128, 12, 8
    W = student_t_weight(5, "gd", m, n)
    nq.nq_set_latent_solver("gd", steps)
    res = nq.nq_lbadmm(W.cuda(), r, iters=iters)
    ref = GD.lbadmm_gd(W.double().numpy(), r=r, iters=iters, steps=steps)
    assert abs(res["rel_err"] - ref.rel_err) <= 0.01 * ref.rel_err
    np.testing.assert_allclose(res["objective"], ref.objective, rtol=0.01)


def test_gd_with_many_steps_approaches_the_exact_update(gd_mode):
    nq = gd_mode
    m, n, r, iters = 512, 384, 64, 6
    W = student_t_weight(6, "gd2", m, n).cuda()
    nq.nq_set_latent_solver("gd", 400)
    gd = nq.nq_lbadmm(W, r, iters=iters)
    nq.nq_set_latent_solver("exact")
    ex = nq.nq_lbadmm(W, r, iters=iters)
    np.testing.assert_allclose(gd["objective"], ex["objective"], rtol=1e-3)
