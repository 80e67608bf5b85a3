"""Pins for the LB-ADMM oracle (CPU only).

Each function of ``oracle.lbadmm`` is checked against something other than itself:
the variational definition of the sub-problem it solves, LAPACK's SVD, scipy's scalar
minimiser, hand-built bit patterns, exhaustive search (C brute force) and the
Eckart-Young bound.
"""
import numpy as np
import pytest
from scipy.optimize import minimize_scalar

from oracle import brute
from oracle.lbadmm import (balance, dual_update, extract_scales, init_latent, latent_update,
                           lbadmm, pack_signs, precondition, recon_error, reconstruct,
                           relative_residual, sign_pm, svid, unpack_signs)
from oracle.splitmix import sign_matrix
from synth import planted_problem


def _augmented(A, X, Y, Z, Lam, rho, lam):
    """The U-step objective written out from its definition."""
    D = A - X @ Y.T
    C = X - Z + Lam
    return 0.5 * np.sum(D * D) + 0.5 * lam * np.sum(X * X) + 0.5 * rho * np.sum(C * C)


@pytest.mark.parametrize("rows,cols,r", [(7, 5, 3), (20, 11, 4), (6, 9, 9)])
def test_latent_update_is_the_minimiser_of_the_augmented_lagrangian(rows, cols, r):
    rng = np.random.default_rng(rows * 100 + r)
    A = rng.standard_normal((rows, cols))
    Y = rng.standard_normal((cols, r))
    Z = rng.standard_normal((rows, r))
    Lam = 0.3 * rng.standard_normal((rows, r))
    rho, lam = 1.3, 0.07
    X, G, R, resid = latent_update(A, Y, Z, Lam, rho, lam)
    assert resid < 1e-10
    f0 = _augmented(A, X, Y, Z, Lam, rho, lam)
    eps = 1e-5
    for _ in range(5):
        E = rng.standard_normal(X.shape)
        fp = _augmented(A, X + eps * E, Y, Z, Lam, rho, lam)
        fm = _augmented(A, X - eps * E, Y, Z, Lam, rho, lam)
        # zero directional derivative, positive curvature
        assert abs(fp - fm) / (2 * eps) < 1e-6 * (1 + abs(f0))
        assert fp > f0 and fm > f0


def test_normal_equations_hold_on_every_solve_of_the_planted_problem():
    p = planted_problem(0, noise=0.1)
    res = lbadmm(p["W"].double().numpy(), r=16, iters=30)
    assert len(res.residuals) == 60
    assert max(res.residuals) < 1e-10


def test_svid_exact_on_rank_one_magnitudes():
    rng = np.random.default_rng(5)
    x = np.exp(rng.standard_normal(9))
    y = np.exp(rng.standard_normal(4))
    S = sign_matrix(3, 9, 4) * np.outer(x, y)
    for K in (1, 3):
        Z, a, b = svid(S, K)
        np.testing.assert_allclose(Z, S, rtol=1e-13)
        np.testing.assert_allclose(np.linalg.norm(a), 1.0, rtol=1e-14)


def test_svid_converges_to_perron_pair():
    rng = np.random.default_rng(6)
    S = rng.standard_normal((30, 8))
    A = np.abs(S)
    Uu, sv, Vt = np.linalg.svd(A)
    u1, v1 = np.abs(Uu[:, 0]), np.abs(Vt[0])
    Z, a, b = svid(S, 200)
    np.testing.assert_allclose(a, u1, atol=1e-10)
    np.testing.assert_allclose(b, sv[0] * v1, rtol=1e-10)
    np.testing.assert_allclose(np.abs(Z), sv[0] * np.outer(u1, v1), rtol=1e-9)
    assert np.all(np.sign(Z) == sign_pm(S))


def test_svid_of_zero_and_dual_identity():
    Z, a, b = svid(np.zeros((3, 2)), 4)
    assert np.all(Z == 0) and np.all(a == 0) and np.all(b == 0)
    rng = np.random.default_rng(7)
    X, Lam = rng.standard_normal((5, 3)), rng.standard_normal((5, 3))
    Zs, _, _ = svid(X + Lam, 4)
    np.testing.assert_allclose(dual_update(Lam, X, Zs), X + Lam - Zs)
    with pytest.raises(ValueError):
        svid(X, 0)


def test_balance_keeps_product_and_equalises_columns():
    rng = np.random.default_rng(8)
    U = rng.standard_normal((12, 4)) * np.array([1.0, 10.0, 0.1, 3.0])
    V = rng.standard_normal((7, 4))
    Ub, Vb, g = balance(U, V)
    np.testing.assert_allclose(Ub @ Vb.T, U @ V.T, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(np.linalg.norm(Ub, axis=0), np.linalg.norm(Vb, axis=0), rtol=1e-13)
    U[:, 2] = 0
    _, _, g = balance(U, V)
    assert g[2] == 1.0


def test_mean_abs_is_the_least_squares_scale_of_the_signs():
    rng = np.random.default_rng(9)
    U = rng.standard_normal((6, 5))
    V = rng.standard_normal((4, 5))
    s1, s2 = extract_scales(U, V, 2.5)
    for i in range(6):
        x = U[i]
        best = minimize_scalar(lambda c: np.sum((x - c * sign_pm(x)) ** 2), bounds=(0, 10),
                               method="bounded", options=dict(xatol=1e-12))
        assert abs(s1[i] / 2.5 - best.x) < 1e-7
    np.testing.assert_allclose(s2, np.abs(V).mean(1))


def test_pack_hand_built_words():
    X = np.ones((2, 33))
    X[0, 0] = -1.0           # bit 0 of word 0
    X[0, 31] = -2.0          # bit 31 of word 0
    X[0, 32] = -0.5          # bit 0 of word 1
    X[1, 5] = -0.0           # negative zero counts as +1
    X[1, 1] = -1e-30
    P = pack_signs(X)
    assert P.dtype == np.uint32 and P.shape == (2, 2)
    assert P[0, 0] == 0x80000001 and P[0, 1] == 0x1
    assert P[1, 0] == 0x2 and P[1, 1] == 0
    assert pack_signs(-np.ones((1, 1)))[0, 0] == 1
    assert pack_signs(-np.ones((1, 31)))[0, 0] == 0x7FFFFFFF
    assert pack_signs(-np.ones((1, 32)))[0, 0] == 0xFFFFFFFF


@pytest.mark.parametrize("r", [1, 31, 32, 33, 100])
def test_pack_round_trip(r):
    rng = np.random.default_rng(r)
    X = rng.standard_normal((9, r))
    np.testing.assert_array_equal(unpack_signs(pack_signs(X), r), sign_pm(X))


def test_recon_error_zero_on_exact_form_and_precondition_scaling():
    rng = np.random.default_rng(10)
    U = sign_matrix(1, 8, 3)
    V = sign_matrix(2, 5, 3)
    s1, s2 = np.exp(rng.standard_normal(8)), np.exp(rng.standard_normal(5))
    W = reconstruct(s1, U, V, s2)
    assert recon_error(W, s1, U, V, s2) < 1e-15
    d_in, d_out = np.exp(rng.standard_normal(5)), np.exp(rng.standard_normal(8))
    Wt, What, gamma = precondition(W, d_in, d_out, r=3)
    np.testing.assert_allclose(Wt, np.diag(d_out) @ W @ np.diag(d_in), rtol=1e-14)
    np.testing.assert_allclose(np.linalg.norm(What), 2.0 * np.sqrt(3), rtol=1e-14)
    np.testing.assert_allclose(What * gamma, Wt, rtol=1e-14)
    Wt0, What0, g0 = precondition(np.zeros((3, 4)), r=2)
    assert g0 == 0.0 and np.all(What0 == 0)


def test_init_latent_scale_and_signs():
    V0 = init_latent(512, 16, 0)
    np.testing.assert_allclose(np.abs(V0), np.sqrt(2.0 / 512))
    np.testing.assert_array_equal(np.sign(V0), sign_matrix(0, 512, 16))


def _match_columns(Us, Up):
    """Max |<u_k, planted_l>|/rows per recovered column and whether it is a signed permutation."""
    M = (Us.T @ Up) / Us.shape[0]
    best = np.abs(M).argmax(axis=1)
    return np.abs(M).max(axis=1), len(set(best.tolist())) == Up.shape[1]


@pytest.mark.parametrize("seed", [0, 1])
def test_planted_factors_recovered_at_zero_noise(seed):
    p = planted_problem(seed, noise=0.0)
    W = p["W"].double().numpy()
    res = lbadmm(W, r=16, iters=100)
    Us, Vs = unpack_signs(res.U_packed, 16), unpack_signs(res.V_packed, 16)
    mu, perm_u = _match_columns(Us, p["U"].numpy())
    mv, perm_v = _match_columns(Vs, p["V"].numpy())
    assert perm_u and perm_v
    assert np.all(mu == 1.0) and np.all(mv == 1.0)        # every sign, up to column sign/order
    assert res.rel_err <= 1e-3


def test_eckart_young_bracket_on_planted_with_noise():
    p = planted_problem(0, noise=0.1)
    W = p["W"].double().numpy()
    rng = np.random.default_rng(0)
    d_in = np.exp(0.5 * rng.standard_normal(W.shape[1]))
    d_out = np.exp(0.5 * rng.standard_normal(W.shape[0]))
    for r in (4, 16):
        res = lbadmm(W, d_in, d_out, r=r, iters=15)
        Wt, _, _ = precondition(W, d_in, d_out, r)
        sv = np.linalg.svd(Wt, compute_uv=False)
        bound = np.sum(sv[r:] ** 2) / np.sum(sv ** 2)
        assert bound <= res.rel_err ** 2 + 1e-12


@pytest.mark.parametrize("shape,r,seed", [((4, 4), 1, 0), ((4, 4), 2, 1), ((6, 6), 1, 2),
                                          ((6, 6), 2, 3), ((5, 6), 2, 4)])
def test_brute_force_lower_bounds_admm(shape, r, seed):
    rng = np.random.default_rng(seed)
    W = rng.standard_normal(shape)
    res = lbadmm(W, r=r, iters=50)
    Wt, _, _ = precondition(W, None, None, r)
    e2_admm = res.rel_err ** 2 * np.sum(Wt * Wt)
    bf, *_ = brute.min_sq_error(Wt, r)
    assert bf <= e2_admm + 1e-9
    # and the ADMM result is a valid instance of the searched family
    Us, Vs = unpack_signs(res.U_packed, r), unpack_signs(res.V_packed, r)
    np.testing.assert_allclose(e2_admm, np.sum((Wt - reconstruct(res.s1, Us, Vs, res.s2)) ** 2),
                               rtol=1e-12)


def test_objective_is_the_latent_relative_residual():
    p = planted_problem(2, noise=0.1)
    W = p["W"].double().numpy()
    seen = {}

    def hook(t, st):
        seen[t] = (st["U"].copy(), st["V"].copy())

    res = lbadmm(W, r=8, iters=3, on_iter=hook)
    _, What, _ = precondition(W, None, None, 8)
    for t in range(3):
        U, V = seen[t]
        direct = np.linalg.norm(What - U @ V.T) ** 2 / np.linalg.norm(What) ** 2
        assert abs(res.objective[t] - direct) < 1e-12
    assert relative_residual(np.zeros((2, 2)), np.ones((2, 1)), np.ones((2, 1))) == 0.0
