"""Pins of the oracle's binary matmul (inference with the packed factors), no GPU.

Checked against things other than its own formula: the reconstruction of the layer from
the same packed factors (identity inputs give its transpose), a rank-one closed form,
the column-sign symmetry of the factorisation, and a word-by-word loop over the packed
bits on tiny inputs.
"""
import numpy as np

from oracle import binary as OB
from oracle import lbadmm as O
from oracle.splitmix import sign_matrix


def _factors(m, n, r, seed):
    rng = np.random.default_rng(seed)
    Us = sign_matrix(seed, m, r)
    Vs = sign_matrix(seed + 1, n, r)
    s1 = np.exp(rng.standard_normal(m))
    s2 = np.exp(rng.standard_normal(n))
    return Us, Vs, O.pack_signs(Us), O.pack_signs(Vs), s1, s2


def test_identity_inputs_give_the_reconstructed_layer():
    m, n, r = 13, 9, 33
    Us, Vs, Up, Vp, s1, s2 = _factors(m, n, r, 3)
    Y = OB.binary_matmul(np.eye(n), Up, Vp, s1, s2, r)
    np.testing.assert_allclose(Y, O.reconstruct(s1, Us, Vs, s2).T, rtol=1e-12, atol=1e-12)


def test_rank_one_all_positive_closed_form():
    m, n = 5, 7
    rng = np.random.default_rng(0)
    s1, s2, X = rng.random(m), rng.random(n), rng.standard_normal((3, n))
    Up = np.zeros((m, 1), dtype=np.uint32)
    Vp = np.zeros((n, 1), dtype=np.uint32)
    Y = OB.binary_matmul(X, Up, Vp, s1, s2, 1)
    np.testing.assert_allclose(Y, np.outer(X @ s2, s1), rtol=1e-12)


def test_flipping_a_rank_column_in_both_factors_changes_nothing():
    m, n, r = 11, 10, 40
    Us, Vs, Up, Vp, s1, s2 = _factors(m, n, r, 5)
    X = np.random.default_rng(1).standard_normal((4, n))
    flip = np.ones(r)
    flip[[0, 31, 32, 39]] = -1
    Y0 = OB.binary_matmul(X, Up, Vp, s1, s2, r)
    Y1 = OB.binary_matmul(X, O.pack_signs(Us * flip), O.pack_signs(Vs * flip), s1, s2, r)
    np.testing.assert_allclose(Y0, Y1, rtol=1e-12, atol=1e-12)


def test_matches_word_loops_on_tiny_inputs():
    m, n, r = 6, 5, 35
    _, _, Up, Vp, s1, s2 = _factors(m, n, r, 9)
    X = np.random.default_rng(2).standard_normal((2, n))
    np.testing.assert_allclose(OB.binary_matmul(X, Up, Vp, s1, s2, r),
                               OB.binary_matmul_loops(X, Up, Vp, s1, s2, r), rtol=1e-12)
