"""Pins of the gradient-descent latent update (oracle/gd.py) to facts it must satisfy.

  * With G a multiple of I (Y = 0) one step lands exactly on the minimiser R / (lam + rho).
  * No step increases f (evaluated from its definition), since eta = 1 / ||G||_inf and
    ||G||_inf bounds G's largest eigenvalue.
  * The distance to the exact minimiser (oracle.lbadmm.latent_update, a Cholesky solve)
    shrinks at least by the factor 1 - lambda_min(G) / ||G||_inf per step, and many steps
    reach it to 1e-10.
  * LB-ADMM with enough steps per half iteration reproduces the exact LB-ADMM.
"""
import numpy as np

from oracle import gd as GD
from oracle import lbadmm as O


def _problem(seed, m=40, n=30, r=6):
    rng = np.random.default_rng(seed)
    A = rng.standard_normal((m, n))
    Y = rng.standard_normal((n, r)) * 0.5
    Z = rng.standard_normal((m, r)) * 0.3
    Lam = rng.standard_normal((m, r)) * 0.3
    X0 = rng.standard_normal((m, r))
    return A, Y, Z, Lam, X0


def test_one_step_is_exact_when_the_gram_is_a_multiple_of_identity():
    A, _, Z, Lam, X0 = _problem(0)
    Y = np.zeros((A.shape[1], 6))
    X, G, R, eta = GD.latent_update_gd(A, Y, Z, Lam, X0, 1.0, 1e-4, 1)
    assert eta == 1.0 / (1.0 + 1e-4)
    np.testing.assert_allclose(X, (Z - Lam) * 1.0 / (1.0 + 1e-4), rtol=0, atol=1e-14)


def test_steps_never_increase_the_objective():
    for seed in range(5):
        A, Y, Z, Lam, X0 = _problem(seed)
        f = [GD.latent_objective(A, X0, Y, Z, Lam, 1.0, 1e-4)]
        X = X0
        for _ in range(30):
            X, _, _, _ = GD.latent_update_gd(A, Y, Z, Lam, X, 1.0, 1e-4, 1)
            f.append(GD.latent_objective(A, X, Y, Z, Lam, 1.0, 1e-4))
        assert all(b <= a + 1e-12 * abs(a) for a, b in zip(f, f[1:]))
        assert f[-1] < f[0]


def test_contraction_towards_the_exact_minimiser():
    for seed in range(5):
        A, Y, Z, Lam, X0 = _problem(seed)
        Xs, G, _, _ = O.latent_update(A, Y, Z, Lam, 1.0, 1e-4)
        q = 1.0 - np.linalg.eigvalsh(G)[0] * GD.gd_step_size(G)
        assert 0.0 < q < 1.0
        d0 = np.linalg.norm(X0 - Xs)
        for k in (1, 5, 20):
            Xk, _, _, _ = GD.latent_update_gd(A, Y, Z, Lam, X0, 1.0, 1e-4, k)
            assert np.linalg.norm(Xk - Xs) <= q ** k * d0 * (1 + 1e-9)
        Xn, _, _, _ = GD.latent_update_gd(A, Y, Z, Lam, X0, 1.0, 1e-4, 3000)
        assert np.max(np.abs(Xn - Xs)) <= 1e-10 * np.max(np.abs(Xs))


def test_lbadmm_with_converged_steps_is_the_exact_lbadmm():
    rng = np.random.default_rng(3)
    W = rng.standard_normal((24, 20))
    ref = O.lbadmm(W, r=4, iters=6, K=4, seed=1)
    got = GD.lbadmm_gd(W, r=4, iters=6, K=4, seed=1, steps=3000)
    np.testing.assert_allclose(got.objective, ref.objective, rtol=1e-8)
    np.testing.assert_allclose(got.s1, ref.s1, rtol=1e-7)
    np.testing.assert_array_equal(got.U_packed, ref.U_packed)
    np.testing.assert_array_equal(got.V_packed, ref.V_packed)
