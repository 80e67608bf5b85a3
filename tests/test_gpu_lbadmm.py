"""GPU parity of LB-ADMM against the FP64 oracle (through the C ABI).

Tolerances:
  * single U (V) step on identical inputs: max|dX| / max|X_ref| <= 2e-3, same for S, a, b;
    a sign of S may differ only where |S_ref| < 1e-3 rms(S_ref).  In the FP32-accurate
    precision mode (split BF16 operands) on FP32 inputs: 1e-4;
  * packing on identical signs: bit-exact;
  * end-to-end reconstruction error within 1% of the oracle's, per instance.
Inputs of the single-step tests are generated here (BF16-exact target and latent operand
for the BF16 mode, FP32 values for the FP32-accurate mode), imported into the GPU state,
and fed unchanged to the oracle.
"""
import numpy as np
import pytest
import torch

from conftest import max_rel
from oracle import calib as OC
from oracle import lbadmm as O
from oracle.splitmix import sign_matrix
from synth import gaussian_weight, planted_problem, stream_tensor

pytestmark = pytest.mark.gpu
TOL_STEP = 2e-3
TOL_STEP_FP32 = 1e-4
TOL_E2E = 0.01


def bf16_exact(a):
    return torch.as_tensor(np.asarray(a), dtype=torch.float32).to(torch.bfloat16).float().numpy()


def unpack(t, r):
    return O.unpack_signs(t.cpu().numpy().view(np.uint32), r)


def test_v0_and_prepare_match_oracle(nq):
    m, n, r = 300, 260, 20
    W = gaussian_weight(3, "W", m, n, 0.02, 0.01, 10.0, torch.float32)
    d_in = torch.exp(0.3 * torch.randn(n))
    d_out = torch.exp(0.3 * torch.randn(m))
    st = nq.LBState(m, n, r)
    gamma = st.prepare(W.cuda(), d_in.cuda(), d_out.cuda(), seed=123)
    Wt, What, g_ref = O.precondition(W.double().numpy(), d_in.double().numpy(),
                                     d_out.double().numpy(), r)
    assert abs(gamma - g_ref) / g_ref < 1e-6
    V = st.field("V")[:, :r].cpu().double().numpy()
    V0 = O.init_latent(n, r, 123)
    np.testing.assert_array_equal(np.sign(V), np.sign(V0))
    np.testing.assert_allclose(V, V0, rtol=1e-7)
    Wh = st.field("WHAT")[:, :n].float().cpu().numpy()
    ref = bf16_exact(What)
    ulp = np.abs(ref) * 2.0 ** -7
    assert np.all(np.abs(Wh - ref) <= ulp + 1e-30)
    assert np.mean(Wh != ref) < 1e-3      # only rounding ties may move by one ulp


@pytest.mark.parametrize("r", [1, 31, 32, 33, 100, 2032])
def test_pack_signs_bit_exact(nq, r):
    rng = np.random.default_rng(r)
    X = rng.standard_normal((77, r)).astype(np.float32)
    X[0, 0] = -0.0
    X[1, :] = 0.0
    X[2, :] = -1e-38
    bits = nq.nq_pack_signs(torch.from_numpy(X).cuda())
    np.testing.assert_array_equal(bits.cpu().numpy().view(np.uint32), O.pack_signs(X))


def _split_bf16(a):
    """hi = bf16(a), lo = bf16(a - hi) of a float32 array (the split operand of the
    FP32-accurate mode)."""
    t = torch.from_numpy(np.asarray(a, dtype=np.float32))
    hi = t.to(torch.bfloat16)
    return hi, (t - hi.float()).to(torch.bfloat16)


def _load_state(st, m, n, r, Wh, U, V, SU, aU, bU, SV, aV, bV):
    hi, lo = _split_bf16(Wh)
    st.field("WHAT")[:, :n].copy_(hi.cuda())
    st.field("WHAT_LO")[:, :n].copy_(lo.cuda())
    for name, val in (("U", U), ("V", V), ("SU", SU), ("SV", SV)):
        st.field(name)[:, :r].copy_(torch.from_numpy(val).float().cuda())
    for name, val in (("AU", aU), ("BU", bU), ("AV", aV), ("BV", bV)):
        st.field(name).copy_(torch.from_numpy(val).float().cuda())
    st.sync_operands()


def _single_step_case(nq, m, n, r, side, seed, rho=1.0, lam=1e-4, K=4, prec="bf16"):
    rng = np.random.default_rng(seed)
    # BF16 mode: BF16-exact target and latent operand (the values its MMAs see);
    # FP32-accurate mode: plain FP32 values
    cast = bf16_exact if prec == "bf16" else (lambda a: np.asarray(a, dtype=np.float32))
    tol = TOL_STEP if prec == "bf16" else TOL_STEP_FP32
    Wh = cast(rng.standard_normal((m, n)) * 0.1)
    U = cast(rng.standard_normal((m, r)) * 0.2).astype(np.float64)
    V = cast(rng.standard_normal((n, r)) * 0.2).astype(np.float64)
    SU = rng.standard_normal((m, r)).astype(np.float32)
    SV = rng.standard_normal((n, r)).astype(np.float32)
    aU, aV = [np.abs(rng.standard_normal(k)).astype(np.float32) / np.sqrt(k) for k in (m, n)]
    bU, bV = [np.abs(rng.standard_normal(r)).astype(np.float32) for _ in range(2)]
    st = nq.LBState(m, n, r, prec=prec)
    st.prepare(torch.zeros(m, n, device="cuda"), seed=0)
    _load_state(st, m, n, r, Wh, U, V, SU, aU, bU, SV, aV, bV)
    st.half_step(side, rho, lam, K)
    assert st.check_device_error() == 0
    A = Wh.astype(np.float64) if side == 0 else Wh.astype(np.float64).T
    Y = V if side == 0 else U
    S0, a0, b0 = (SU, aU, bU) if side == 0 else (SV, aV, bV)
    S0 = S0.astype(np.float64)
    Z = O.sign_pm(S0) * np.outer(a0, b0)
    Lam = S0 - Z
    Xr, _, _, _ = O.latent_update(A, Y, Z, Lam, rho, lam)
    Sr = Xr + Lam
    _, ar, br = O.svid(Sr, K)
    tag = "U" if side == 0 else "V"
    X = st.field(tag)[:, :r].cpu().double().numpy()
    S = st.field("S" + tag)[:, :r].cpu().double().numpy()
    a = st.field("A" + tag).cpu().double().numpy()
    b = st.field("B" + tag).cpu().double().numpy()
    assert max_rel(X, Xr) <= tol
    assert max_rel(S, Sr) <= tol
    assert max_rel(a, ar) <= tol
    assert max_rel(b, br) <= tol
    flips = np.sign(S) != np.sign(Sr)
    rms = np.sqrt(np.mean(Sr ** 2))
    assert np.all(np.abs(Sr[flips]) < 1e-3 * rms)
    # normal-equation residual of the GPU's solve: ||X G - R|| / ||R|| with the exact
    # G = Y^T Y + (lambda + rho) I and R of these inputs (the solve's own accuracy)
    G = Y.T @ Y + (lam + rho) * np.eye(r)
    R = A @ Y + rho * (Z - Lam)
    resid = float(np.linalg.norm(X @ G - R) / np.linalg.norm(R))
    assert resid <= 1e-4, resid
    # the transposed BF16 operand the other side will read
    xt_ref = bf16_exact(Xr)
    return max_rel(X, Xr), st, xt_ref


@pytest.mark.parametrize("m,n,r", [(300, 200, 40), (1000, 777, 130), (520, 600, 300),
                                   (129, 65, 1), (256, 512, 16), (700, 900, 257)])
@pytest.mark.parametrize("side", [0, 1])
def test_single_step_matches_oracle(nq, m, n, r, side):
    _single_step_case(nq, m, n, r, side, seed=m + n + r + side)


@pytest.mark.parametrize("m,n,r", [(300, 200, 40), (520, 600, 300), (129, 65, 1),
                                   (256, 512, 16)])
@pytest.mark.parametrize("side", [0, 1])
def test_single_step_fp32_precision_matches_oracle(nq, m, n, r, side):
    _single_step_case(nq, m, n, r, side, seed=3 * m + n + r + side, prec="fp32")


@pytest.mark.parametrize("m,n,r", [(11008, 4096, 1000), (8192, 8192, 4080), (28672, 8192, 3488)])
@pytest.mark.parametrize("side", [0, 1])
def test_single_step_large_shapes(nq, m, n, r, side):
    # the 11008 x 4096 r = 1000 target layer, config 5's largest rank (64 Cholesky block
    # steps) and config 4's 70B gate/up shape (non-square, r = 3488)
    err, _, _ = _single_step_case(nq, m, n, r, side, seed=m + r + side)
    assert err < TOL_STEP


def test_single_step_full_size_q_proj(nq):
    # Llama-2-7B q_proj shape at 1 BPW (4096 x 4096, r = 2032): both sides
    for side in (0, 1):
        err, _, _ = _single_step_case(nq, 4096, 4096, 2032, side, seed=7 + side)
        assert err < TOL_STEP


def test_planted_factors_recovered_on_gpu(nq):
    p = planted_problem(0, noise=0.0)
    res = nq.nq_lbadmm(p["W"].cuda(), 16, iters=100)
    Us, Vs = unpack(res["U_packed"], 16), unpack(res["V_packed"], 16)
    for got, planted in ((Us, p["U"].numpy()), (Vs, p["V"].numpy())):
        M = np.abs(got.T @ planted) / got.shape[0]
        assert np.all(M.max(axis=1) == 1.0)
        assert len(set(M.argmax(axis=1).tolist())) == 16
    assert res["rel_err"] <= 1e-3


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_planted_with_noise_end_to_end(nq, seed):
    # Identity preconditioners, 60 iterations: the iteration has converged and the final
    # error is a well-defined value; per instance within 1 % of the oracle.  (At 30
    # iterations this problem is bistable, see test_config1_statistics_at_thirty_iterations.)
    p = planted_problem(seed, noise=0.1)
    res = nq.nq_lbadmm(p["W"].cuda(), 16, iters=60)
    ref = O.lbadmm(p["W"].double().numpy(), r=16, iters=60)
    assert abs(res["rel_err"] - ref.rel_err) <= TOL_E2E * ref.rel_err, (res["rel_err"], ref.rel_err)
    # the first objective values: identical start, FP32-accurate arithmetic
    np.testing.assert_allclose(res["objective"][:5], ref.objective[:5], rtol=1e-4)


def test_config1_statistics_at_thirty_iterations(nq):
    # The first benchmark configuration as stated: 256 x 512 FP32 planted r = 16 with 0.1
    # noise, calibration preconditioners from 4096-token act/grad streams, 30 iterations.
    # At 30 iterations the iteration is still in a transient whose outcome moves by 1-3 %
    # under state perturbations of 1e-6 (relative) - the FP64 oracle's own outcome does -
    # so no arithmetic short of the oracle's own operation order reproduces one instance
    # to 1 %.  Read statistically over 64 seeds: the median and the 90th percentile of
    # the GPU's final errors each lie within 1 % of the oracle's, and every instance's
    # first-iteration objective (identical start) agrees to 1e-4.
    e_gpu, e_ref = [], []
    for seed in range(64):
        p = planted_problem(seed, noise=0.1)
        d_in, d_out, _, _ = nq.nq_calib_precond(p["acts"].cuda(), p["grads"].cuda())
        res = nq.nq_lbadmm(p["W"].cuda(), 16, d_in, d_out, iters=30)
        r_in, r_out, _, _ = OC.calib_precond([p["acts"].numpy()], [p["grads"].numpy()])
        ref = O.lbadmm(p["W"].double().numpy(), r_in, r_out, r=16, iters=30)
        assert abs(res["objective"][0] - ref.objective[0]) <= 1e-4 * ref.objective[0]
        e_gpu.append(res["rel_err"])
        e_ref.append(ref.rel_err)
    for q in (50, 90):
        g, o = np.percentile(e_gpu, q), np.percentile(e_ref, q)
        assert abs(g - o) <= TOL_E2E * o, (q, g, o)


def test_random_layer_end_to_end_within_one_percent(nq):
    # 2048 x 2048 BF16 layer with 1% outlier input columns, calibration streams of 8192
    # tokens, 1 BPW (r = 1008), 20 iterations: large enough for the error to self-average.
    m = n = 2048
    r = 1008
    W = gaussian_weight(5, "W", m, n, 0.02, 0.01, 10.0)
    acts = stream_tensor(5, "acts", 8192, n)
    grads = stream_tensor(5, "grads", 8192, m)
    d_in, d_out, _, _ = nq.nq_calib_precond(acts.cuda(), grads.cuda())
    res = nq.nq_lbadmm(W.cuda(), r, d_in, d_out, iters=20)
    r_in, r_out, _, _ = OC.calib_precond([acts.float().numpy()], [grads.float().numpy()])
    Wd = W.double().numpy()
    ref = O.lbadmm(Wd, r_in, r_out, r=r, iters=20)
    assert abs(res["rel_err"] - ref.rel_err) <= TOL_E2E * ref.rel_err, (res["rel_err"], ref.rel_err)
    # Eckart-Young: no rank-r matrix beats the truncated SVD
    Wt, _, _ = O.precondition(Wd, r_in, r_out, r)
    sv = np.linalg.svd(Wt, compute_uv=False)
    assert np.sum(sv[r:] ** 2) / np.sum(sv ** 2) <= res["rel_err"] ** 2
    # the dedicated entry point agrees with the error nq_lbadmm reported
    e2 = nq.nq_recon_error(W.cuda(), res["U_packed"], res["V_packed"], r, res["s1"], res["s2"],
                           d_in, d_out)
    assert abs(e2 - res["rel_err"]) <= 1e-5 * res["rel_err"]


@pytest.mark.parametrize("m,n,r", [(257, 300, 33), (64, 1000, 7)])
def test_recon_error_entry_matches_oracle(nq, m, n, r):
    rng = np.random.default_rng(m)
    W = rng.standard_normal((m, n)).astype(np.float32)
    Us = sign_matrix(1, m, r)
    Vs = sign_matrix(2, n, r)
    s1 = np.exp(rng.standard_normal(m)).astype(np.float32)
    s2 = np.exp(rng.standard_normal(n)).astype(np.float32) / r
    d_in = np.exp(0.2 * rng.standard_normal(n)).astype(np.float32)
    d_out = np.exp(0.2 * rng.standard_normal(m)).astype(np.float32)
    Up = torch.from_numpy(O.pack_signs(Us).view(np.int32)).cuda()
    Vp = torch.from_numpy(O.pack_signs(Vs).view(np.int32)).cuda()
    e = nq.nq_recon_error(torch.from_numpy(W).cuda(), Up, Vp, r, torch.from_numpy(s1).cuda(),
                          torch.from_numpy(s2).cuda(), torch.from_numpy(d_in).cuda(),
                          torch.from_numpy(d_out).cuda())
    Wt = (d_out[:, None].astype(np.float64) * W) * d_in[None, :]
    ref = O.recon_error(Wt, s1.astype(np.float64), Us, Vs, s2.astype(np.float64))
    assert abs(e - ref) <= 1e-5 * ref


def test_zero_weight_is_a_fixed_point(nq):
    res = nq.nq_lbadmm(torch.zeros(200, 100, device="cuda"), 8, iters=3)
    assert res["rel_err"] == 0.0
    assert torch.all(res["s1"] == 0) and torch.all(res["s2"] == 0)
    assert torch.all(res["U_packed"] == 0) and torch.all(res["V_packed"] == 0)
    assert all(o == 0.0 for o in res["objective"])


def test_nonfinite_weight_is_reported(nq):
    W = torch.randn(128, 96)
    W[5, 7] = float("inf")
    with pytest.raises(nq.NQError) as e:
        nq.nq_lbadmm(W.cuda(), 8, iters=2)
    assert e.value.code == 4


def test_runs_are_bit_identical(nq):
    W = gaussian_weight(9, "W", 640, 384, dtype=torch.bfloat16).cuda()
    a = nq.nq_lbadmm(W, 96, iters=5)
    b = nq.nq_lbadmm(W, 96, iters=5)
    assert torch.equal(a["U_packed"], b["U_packed"]) and torch.equal(a["V_packed"], b["V_packed"])
    assert torch.equal(a["s1"], b["s1"]) and torch.equal(a["s2"], b["s2"])
    assert a["objective"] == b["objective"] and a["rel_err"] == b["rel_err"]


def test_full_size_q_proj_pipeline_properties(nq):
    # The bench workload: 4096 x 4096 BF16 q_proj with 1% x10 outlier columns, 262144-token
    # act/grad streams, r = 2032 (1 BPW), 100 iterations.  The oracle cannot run 100
    # iterations at this size within a test; checked here: Eckart-Young, agreement of the
    # two error paths, a decreasing objective, and balanced-scale consistency.
    m = n = 4096
    r = nq.nq_rank_for_bpw(m, n, 1.0)
    assert r == 2032
    W = gaussian_weight(0, "W", m, n, 0.02, 0.01, 10.0).cuda()
    acts = stream_tensor(0, "acts", 262144, n).cuda()
    grads = stream_tensor(0, "grads", 262144, m).cuda()
    d_in, d_out, _, _ = nq.nq_calib_precond(acts, grads)
    del acts, grads
    res = nq.nq_lbadmm(W, r, d_in, d_out, iters=100)
    e = res["rel_err"]
    obj = res["objective"]
    assert np.isfinite(e) and 0 < e < 1
    assert obj[-1] < obj[0]
    Wt = (d_out.double()[:, None] * W.double() * d_in.double()[None, :]).cpu().numpy()
    ev = np.linalg.eigvalsh(Wt.T @ Wt)[::-1]
    assert np.sum(ev[r:]) / np.sum(ev) <= e ** 2
    e2 = nq.nq_recon_error(W, res["U_packed"], res["V_packed"], r, res["s1"], res["s2"],
                           d_in, d_out)
    assert abs(e2 - e) <= 1e-5 * e
    assert torch.all(res["s1"] > 0) and torch.all(res["s2"] > 0)


def _late_state(m, n, r, seed, eps, cast):
    """A state late in a run: W^ = c (A B^T + eps sqrt(r) N) with ||W^|| = 2 sqrt(r) (the
    library's normalisation), latents U = sqrt(c) A, V = sqrt(c) B (U V^T fits W^ up to
    the noise, a relative residual of about eps^2), S = latent + 0.05 N, positive a, b."""
    rng = np.random.default_rng(seed)
    A = rng.standard_normal((m, r))
    B = rng.standard_normal((n, r))
    M = A @ B.T + eps * np.sqrt(r) * rng.standard_normal((m, n))
    c = 2 * np.sqrt(r) / np.linalg.norm(M)
    Wh = cast(c * M)
    U, V = cast(np.sqrt(c) * A).astype(np.float64), cast(np.sqrt(c) * B).astype(np.float64)
    SU = (U + 0.05 * rng.standard_normal((m, r))).astype(np.float32)
    SV = (V + 0.05 * rng.standard_normal((n, r))).astype(np.float32)
    aU, aV = [np.abs(rng.standard_normal(k)).astype(np.float32) / np.sqrt(k) for k in (m, n)]
    bU, bV = [0.1 * np.abs(rng.standard_normal(r)).astype(np.float32) for _ in range(2)]
    return Wh, U, V, SU, aU, bU, SV, aV, bV


def _oracle_iteration(Wh, U, V, SU, aU, bU, SV, aV, bV, rho=1.0, lam=1e-4, operand=None):
    """The U and V steps of one iteration from the loaded state; ``operand`` (if given)
    rounds U before the V step takes it as its contraction operand, as the BF16 mode
    defines it."""
    W = Wh.astype(np.float64)
    ZU = O.sign_pm(SU) * np.outer(aU, bU)
    LU = SU.astype(np.float64) - ZU
    ZV = O.sign_pm(SV) * np.outer(aV, bV)
    LV = SV.astype(np.float64) - ZV
    U1, _, _, _ = O.latent_update(W, V, ZU, LU, rho, lam)
    if operand is not None:
        U1 = operand(U1).astype(np.float64)
    V1, _, _, _ = O.latent_update(W.T, U1, ZV, LV, rho, lam)
    return U1, V1


@pytest.mark.parametrize("prec,m,n,r,eps", [("fp32", 2048, 2048, 1008, 0.05),
                                            ("bf16", 4096, 4096, 2032, 0.05),
                                            ("bf16", 4096, 4096, 2032, 0.3)])
def test_objective_on_identical_late_state(nq, prec, m, n, r, eps):
    # The per-iteration objective (||W^||^2 - 2 <W^T U, V> + <U^T U, V^T V>) / ||W^||^2
    # subtracts terms near ||W^||^2 when the residual is small (eps = 0.05: ~6e-4 after
    # one step).  From an identical late state (rho = 1e-3, so that the step fits W^):
    # one iteration on the GPU, then its objective (i) against the explicit residual of
    # W^ and the GPU's U, V as its operands hold them (BF16-rounded in the BF16 mode):
    # 1e-4 relative plus the accumulation floor below, the formula's own accuracy;
    # (ii) against the oracle's iteration from the same state, with the latents rounded
    # where the BF16 mode rounds them: 1e-3 relative plus the same floor.
    rho, lam = 1e-3, 1e-4
    cast = bf16_exact if prec == "bf16" else (lambda a: np.asarray(a, dtype=np.float32))
    Wh, U, V, SU, aU, bU, SV, aV, bV = _late_state(m, n, r, 5, eps, cast)
    st = nq.LBState(m, n, r, prec=prec)
    # prepare on W^ itself: ||W^|| = 2 sqrt(r), so gamma = 1 and W^ and its norm are
    # formed as they will be loaded
    Wt = torch.from_numpy(Wh).to(torch.bfloat16 if prec == "bf16" else torch.float32)
    st.prepare(Wt.cuda(), seed=0)
    _load_state(st, m, n, r, Wh, U, V, SU, aU, bU, SV, aV, bV)
    obj = st.iterate(1, rho=rho, lam=lam)[0]
    assert st.check_device_error() == 0
    U1 = st.field("U")[:, :r].cpu().double().numpy()
    V1 = st.field("V")[:, :r].cpu().double().numpy()
    Wd = Wh.astype(np.float64)
    op = bf16_exact if prec == "bf16" else (lambda a: a)
    explicit = O.relative_residual(Wd, op(U1).astype(np.float64), op(V1).astype(np.float64))
    # Each term of the identity is about ||W^||^2 and reaches the difference through FP32
    # tensor-core accumulation over K <= 4096 products: about 4 * 2^-24 * sqrt(K) of
    # ||W^||^2 apiece, so the objective carries an absolute floor of ~2e-5 (margin 5e-5)
    # besides its relative 1e-4.
    floor = 5e-5
    assert abs(obj - explicit) <= 1e-4 * explicit + floor, (obj, explicit)
    U1r, V1r = _oracle_iteration(Wh, U, V, SU, aU, bU, SV, aV, bV, rho=rho, lam=lam,
                                 operand=bf16_exact if prec == "bf16" else None)
    ref = O.relative_residual(Wd, U1r, op(V1r).astype(np.float64))
    assert abs(obj - ref) <= 1e-3 * ref + floor, (obj, ref)


@pytest.mark.parametrize("m,n,r", [(300, 500, 40), (4096, 4096, 2032), (777, 1000, 33)])
def test_finish_scales_and_bits_on_loaded_latents(nq, m, n, r):
    # balancing, scale extraction and packing on identical latents: s1, s2 within 1e-5 of
    # the oracle, packed words bit for bit
    rng = np.random.default_rng(m + r)
    W = torch.randn(m, n, generator=torch.Generator().manual_seed(r)) * 0.02
    st = nq.LBState(m, n, r, prec="fp32")
    gamma = st.prepare(W.cuda(), seed=0)
    U = (rng.standard_normal((m, r)) * np.exp(rng.standard_normal(r))).astype(np.float32)
    V = (rng.standard_normal((n, r)) * np.exp(rng.standard_normal(r))).astype(np.float32)
    U[3, 5 % r] = 0.0
    st.field("U")[:, :r].copy_(torch.from_numpy(U).cuda())
    st.field("V")[:, :r].copy_(torch.from_numpy(V).cuda())
    res = st.finish(W.cuda())
    Ub, Vb, _ = O.balance(U.astype(np.float64), V.astype(np.float64))
    s1, s2 = O.extract_scales(Ub, Vb, gamma)
    assert max_rel(res["s1"].cpu().numpy(), s1) <= 1e-5
    assert max_rel(res["s2"].cpu().numpy(), s2) <= 1e-5
    np.testing.assert_array_equal(res["U_packed"].cpu().numpy().view(np.uint32), O.pack_signs(Ub))
    np.testing.assert_array_equal(res["V_packed"].cpu().numpy().view(np.uint32), O.pack_signs(Vb))
    Wt, _, _ = O.precondition(W.double().numpy(), None, None, r)
    ref = O.recon_error(Wt, s1, O.sign_pm(Ub), O.sign_pm(Vb), s2)
    assert abs(res["rel_err"] - ref) <= 1e-5 * ref


@pytest.mark.parametrize("shape,r,seed", [((4, 4), 1, 0), ((4, 4), 2, 1), ((6, 6), 1, 2),
                                          ((6, 6), 2, 3), ((6, 6), 2, 4)])
def test_brute_force_lower_bounds_the_gpu_result(nq, shape, r, seed):
    # Exhaustive search over every sign pattern with least-squares scales lower-bounds
    # the squared error of any factorisation of this family, the GPU's included.
    from oracle import brute
    W = np.random.default_rng(seed).standard_normal(shape)
    res = nq.nq_lbadmm(torch.from_numpy(W.astype(np.float32)).cuda(), r, iters=50)
    Wt, _, _ = O.precondition(W.astype(np.float32).astype(np.float64), None, None, r)
    e2_gpu = res["rel_err"] ** 2 * np.sum(Wt * Wt)
    bf, *_ = brute.min_sq_error(Wt, r)
    assert bf <= e2_gpu * (1 + 1e-6) + 1e-12, (bf, e2_gpu)
