"""GPU checks of the Newton-Schulz update of G^-1 (nq_set_inverse_mode) against the oracle.

The update replaces the r x r factorisation of a half step when the side's previous
inverse is a close start: X_{k+1} = X_k + (I - X_k G) X_k, accepted once
||I - X_k G||_F <= 1e-2, so that ||I - X G||_2 <= 1e-4 plus rounding.  Its rounding
floor (split-BF16 products; emulated in FP64 on the Grams of an oracle run of the
11008 x 4096 layer at r = 1000, condition numbers 5-20) is ||I - X G||_2 ~ 1e-4, about
twice the Cholesky path's 6e-5.  Tolerances:
  * BF16 mode single step: the same 2e-3 as the Cholesky path (the operand rounding,
    4e-3 relative per entry, dominates the inverse's 1e-4);
  * FP32-accurate mode single step: 2e-4 of max|X| and a normal-equation residual of
    3e-4 (twice the Cholesky path's 1e-4, from the floor above);
  * a failed update falls back to the Cholesky path: bit-identical to that path;
  * over a run: the update is accepted on at least 80 % of the attempts, and the final
    reconstruction error is within 1 % of the Cholesky-only run's.
"""
import numpy as np
import pytest
import torch

from conftest import max_rel
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
def modes(nq):
    yield nq
    nq.nq_set_inverse_mode("auto")
    nq.nq_set_tuning("newton_fused", 0)


def _state(nq, m, n, r, prec, seed):
    rng = np.random.default_rng(seed)
    cast = bf16_exact if prec == "bf16" else (lambda a: np.asarray(a, dtype=np.float32))
    Wh = cast(rng.standard_normal((m, n)) * 0.1)
    U = cast(rng.standard_normal((m, r)) * 0.2).astype(np.float64)
    V = cast(rng.standard_normal((n, r)) * 0.2).astype(np.float64)
    SU = rng.standard_normal((m, r)).astype(np.float32)
    SV = rng.standard_normal((n, r)).astype(np.float32)
    aU, aV = [np.abs(rng.standard_normal(k)).astype(np.float32) / np.sqrt(k) for k in (m, n)]
    bU, bV = [np.abs(rng.standard_normal(r)).astype(np.float32) for _ in range(2)]
    return dict(Wh=Wh, U=U, V=V, SU=SU, SV=SV, aU=aU, aV=aV, bU=bU, bV=bV, rng=rng)


def _load(nq, m, n, r, prec, d, start):
    """A workspace holding state ``d`` with ``start`` as the previous G^-1 of both sides."""
    st = nq.LBState(m, n, r, prec=prec)
    st.prepare(torch.zeros(m, n, device="cuda"), seed=0)
    hi, lo = _split(d["Wh"])
    st.field("WHAT")[:, :n].copy_(hi.cuda())
    st.field("WHAT_LO")[:, :n].copy_(lo.cuda())
    for name in ("U", "V", "SU", "SV"):
        st.field(name)[:, :r].copy_(torch.from_numpy(d[name]).float().cuda())
    for name, key in (("AU", "aU"), ("BU", "bU"), ("AV", "aV"), ("BV", "bV")):
        st.field(name).copy_(torch.from_numpy(d[key]).float().cuda())
    st.sync_operands()
    for side, X0 in start.items():
        nm = "GINV_U" if side == 0 else "GINV_V"
        h, l = _split(X0)
        st.field(nm)[:r, :r].copy_(h.cuda())
        st.field(nm + "_LO")[:r, :r].copy_(l.cuda())
    torch.cuda.synchronize()
    return st


def _gram(d, side, r, lam=1e-4, rho=1.0):
    Y = d["V"] if side == 0 else d["U"]
    return Y.T @ Y + (lam + rho) * np.eye(r), Y


def _perturbed_inverse(G, eps, rng):
    """A symmetric start X_0 with ||I - X_0 G||_2 about eps."""
    r = G.shape[0]
    P = rng.standard_normal((r, r))
    P = (P + P.T) / 2
    P *= eps / np.linalg.norm(P, 2)
    Gi = np.linalg.inv(G)
    return Gi + Gi @ P @ Gi / np.linalg.norm(Gi, 2)


@pytest.mark.parametrize("prec,m,n,r", [("bf16", 1000, 777, 300), ("bf16", 700, 900, 257),
                                        ("fp32", 520, 600, 300), ("bf16", 2048, 1536, 1000)])
@pytest.mark.parametrize("side", [0, 1])
@pytest.mark.parametrize("fused", [0, 1])
def test_newton_single_step_matches_oracle(modes, prec, m, n, r, side, fused):
    # both forms of the update: two launches per step, and all steps in one launch
    nq = modes
    nq.nq_set_tuning("newton_fused", fused)
    rho, lam, K = 1.0, 1e-4, 4
    d = _state(nq, m, n, r, prec, seed=11 * m + r + side)
    G, Y = _gram(d, side, r, lam, rho)
    X0 = _perturbed_inverse(G, 0.3, d["rng"])
    st = _load(nq, m, n, r, prec, d, {side: X0})
    nq.nq_set_inverse_mode("newton")
    st.half_step(side, rho, lam, K)
    assert st.check_device_error() == 0
    stats = st.inv_stats()
    assert stats["accepted"] == 1 and stats["fallbacks"] == 0, stats
    assert 3 <= stats["steps"] <= 6, stats
    # the accepted inverse against the exact one of the Gram the GPU formed (of the
    # operands as held: BF16, or hi + lo in the FP32-accurate mode)
    Xg = st.ginv(side).cpu().double().numpy()
    resid = np.linalg.norm(np.eye(r) - Xg @ G, 2)
    assert resid <= (5e-4 if prec == "bf16" else 3e-4), resid
    # the step's result against the oracle's exact solve
    A = d["Wh"].astype(np.float64) if side == 0 else d["Wh"].astype(np.float64).T
    S0, a0, b0 = (d["SU"], d["aU"], d["bU"]) if side == 0 else (d["SV"], d["aV"], d["bV"])
    S0 = S0.astype(np.float64)
    Z = O.sign_pm(S0) * np.outer(a0, b0)
    Lam = S0 - Z
    Xr, _, R, _ = O.latent_update(A, Y, Z, Lam, rho, lam)
    tag = "U" if side == 0 else "V"
    X = st.field(tag)[:, :r].cpu().double().numpy()
    tol = 2e-3 if prec == "bf16" else 2e-4
    assert max_rel(X, Xr) <= tol
    ne = float(np.linalg.norm(X @ G - R) / np.linalg.norm(R))
    assert ne <= (1e-3 if prec == "bf16" else 3e-4), ne


@pytest.mark.parametrize("prec", ["bf16", "fp32"])
@pytest.mark.parametrize("fused", [0, 1])
def test_failed_update_falls_back_to_cholesky_bit_for_bit(modes, prec, fused):
    nq = modes
    nq.nq_set_tuning("newton_fused", fused)
    m, n, r, side = 600, 500, 320, 0
    d = _state(nq, m, n, r, prec, seed=5)
    G, _ = _gram(d, side, r)
    # X_0 = 3 G^-1: E_0 = -2 I, the iteration diverges and is dropped after one step
    st = _load(nq, m, n, r, prec, d, {side: 3.0 * np.linalg.inv(G)})
    nq.nq_set_inverse_mode("newton")
    st.half_step(side)
    assert st.check_device_error() == 0
    stats = st.inv_stats()
    assert stats["accepted"] == 0 and stats["fallbacks"] == 1, stats
    X_nt = st.field("U")[:, :r].clone()
    S_nt = st.field("SU")[:, :r].clone()
    ref = _load(nq, m, n, r, prec, d, {})
    nq.nq_set_inverse_mode("cholesky")
    ref.half_step(side)
    assert ref.check_device_error() == 0
    assert torch.equal(X_nt, ref.field("U")[:, :r])
    assert torch.equal(S_nt, ref.field("SU")[:, :r])
    assert ref.inv_stats()["accepted"] == 0 and ref.inv_stats()["fallbacks"] == 0


def test_zero_start_falls_back(modes):
    # right after prepare the previous inverses are zero: X_1 = X_0 = 0, E does not shrink
    nq = modes
    m, n, r = 700, 600, 300
    W = student_t_weight(3, "w", m, n).cuda()
    st = nq.LBState(m, n, r)
    st.prepare(W)
    nq.nq_set_inverse_mode("newton")
    st.iterate(1, want_objective=False)
    assert st.check_device_error() == 0
    s = st.inv_stats()
    assert s["accepted"] == 0 and s["fallbacks"] == 2, s


@pytest.mark.parametrize("m,n,r,iters,fused", [(2752, 1024, 320, 16, 0), (11008, 4096, 1000, 12, 0),
                                               (11008, 4096, 1000, 12, 1), (4096, 4096, 2032, 12, 1)])
def test_auto_mode_run_matches_cholesky_run(modes, m, n, r, iters, fused):
    nq = modes
    nq.nq_set_tuning("newton_fused", fused)
    W = student_t_weight(0, "gate", m, n).cuda()
    res = {}
    for mode in ("cholesky", "auto"):
        nq.nq_set_inverse_mode(mode)
        st = nq.LBState(m, n, r)
        st.prepare(W)
        obj = st.iterate(iters)
        out = st.finish(W)
        res[mode] = (np.array(obj), out["rel_err"], st.inv_stats())
    o_c, e_c, s_c = res["cholesky"]
    o_a, e_a, s_a = res["auto"]
    first = 4 if r > 1536 else 3          # the auto mode's first attempt
    attempts = 2 * (iters - first)
    assert s_c["accepted"] == 0 and s_c["fallbacks"] == 0
    assert s_a["accepted"] + s_a["fallbacks"] == attempts, s_a
    assert s_a["accepted"] >= 0.8 * attempts, s_a
    # identical up to the first attempt, then the same trajectory to rounding
    np.testing.assert_array_equal(o_a[:first], o_c[:first])
    assert np.max(np.abs(o_a - o_c) / o_c) <= 1e-2
    assert abs(e_a - e_c) <= 0.01 * e_c
