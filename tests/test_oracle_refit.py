"""Pins of the oracle's least-squares scale refit (no GPU).

Checked against properties fixed by the mathematics: the error never increases; at the
refit's fixed point the gradient of the squared error with respect to every scale
vanishes; a planted diag(a) P diag(b) is recovered exactly (error 0) from perturbed
scales; and on one row with one column the update is the scalar least-squares ratio.
"""
import numpy as np

from oracle import lbadmm as O
from oracle import refit as R
from oracle.splitmix import sign_matrix


def _problem(m, n, r, seed, planted=False):
    rng = np.random.default_rng(seed)
    Us, Vs = sign_matrix(seed, m, r), sign_matrix(seed + 1, n, r)
    a, b = np.exp(0.5 * rng.standard_normal(m)), np.exp(0.5 * rng.standard_normal(n))
    W = (a[:, None] * (Us @ Vs.T)) * b[None, :]
    if not planted:
        W = W + 0.3 * rng.standard_normal((m, n)) * np.sqrt(np.mean(W * W))
    return W, Us, Vs, a, b


def test_error_never_increases():
    W, Us, Vs, _, _ = _problem(40, 30, 7, 1)
    Ub, Vb, _ = O.balance(Us * 0.9, Vs * 1.1)
    s1, s2 = O.extract_scales(Ub, Vb, 1.0)
    _, _, errors = R.ls_refit(W, Us, Vs, s1, s2, sweeps=6)
    assert all(e1 <= e0 + 1e-15 for e0, e1 in zip(errors, errors[1:]))
    assert errors[-1] < errors[0]


def test_fixed_point_has_zero_gradient():
    W, Us, Vs, _, _ = _problem(25, 35, 5, 2)
    s1, s2, _ = R.ls_refit(W, Us, Vs, np.ones(25), np.ones(35), sweeps=400)
    P = Us @ Vs.T
    D = W - (s1[:, None] * P) * s2[None, :]
    g1 = -(D * P) @ s2            # d/ds1 of ||D||^2 / 2
    g2 = -(D * P).T @ s1
    scale = np.linalg.norm(W) * max(np.abs(s1).max(), np.abs(s2).max())
    assert np.abs(g1).max() < 1e-8 * scale and np.abs(g2).max() < 1e-8 * scale


def test_planted_scales_are_recovered_exactly():
    W, Us, Vs, a, b = _problem(20, 24, 6, 3, planted=True)
    rng = np.random.default_rng(0)
    s1, s2, errors = R.ls_refit(W, Us, Vs, a * np.exp(0.1 * rng.standard_normal(20)),
                                b * np.exp(0.1 * rng.standard_normal(24)), sweeps=200)
    assert errors[-1] < 1e-10


def test_single_entry_is_the_scalar_ratio():
    # one row and one column, r = 3 with P = +1 + 1 - 1 = 1: s1 <- w / (p s2) ... exactly
    Us = np.array([[1.0, 1.0, -1.0]])
    Vs = np.array([[1.0, 1.0, 1.0]])
    s1, s2, errors = R.ls_refit(np.array([[6.0]]), Us, Vs, np.array([1.0]), np.array([2.0]),
                                sweeps=1)
    assert s1[0] == 3.0 and s2[0] == 2.0 and errors[-1] == 0.0
