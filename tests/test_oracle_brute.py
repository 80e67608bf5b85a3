"""Pins for the C brute-force enumerator itself (CPU only)."""
import numpy as np
import pytest

from oracle import brute
from oracle.splitmix import sign_matrix


@pytest.mark.parametrize("shape,seed", [((4, 4), 0), ((6, 6), 1), ((3, 7), 2)])
def test_rank_one_is_the_best_rank_one_approximation(shape, seed):
    # With real scales every +-1 pattern spans all rank-1 matrices, so the optimum is
    # ||W||^2 - sigma_1^2 (Eckart-Young, LAPACK SVD).
    W = np.random.default_rng(seed).standard_normal(shape)
    sv = np.linalg.svd(W, compute_uv=False)
    e, U, V, s1, s2 = brute.min_sq_error(W, 1)
    assert abs(e - (np.sum(W * W) - sv[0] ** 2)) < 1e-9


def test_planted_rank_two_is_found_exactly():
    rng = np.random.default_rng(3)
    U = sign_matrix(11, 6, 2)
    V = sign_matrix(12, 6, 2)
    W = (np.exp(rng.standard_normal(6))[:, None] * (U @ V.T)) * np.exp(rng.standard_normal(6))[None, :]
    e, Ub, Vb, s1, s2 = brute.min_sq_error(W, 2)
    assert e < 1e-18 * np.sum(W * W) + 1e-20
    np.testing.assert_allclose((s1[:, None] * (Ub @ Vb.T)) * s2[None, :], W, atol=1e-9)


@pytest.mark.parametrize("seed", [4, 5])
def test_rank_two_respects_eckart_young(seed):
    W = np.random.default_rng(seed).standard_normal((6, 6))
    sv = np.linalg.svd(W, compute_uv=False)
    e, *_ = brute.min_sq_error(W, 2)
    assert e >= np.sum(sv[2:] ** 2) - 1e-9
    e1, *_ = brute.min_sq_error(W, 1)
    assert e <= e1 + 1e-9


def test_rejects_unsupported_sizes():
    with pytest.raises(ValueError):
        brute.min_sq_error(np.zeros((9, 2)), 1)
    with pytest.raises(ValueError):
        brute.min_sq_error(np.zeros((3, 3)), 3)
