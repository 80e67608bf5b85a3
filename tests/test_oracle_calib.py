"""Pins for the oracle's calibration statistics and Ledoit-Wolf preconditioners (CPU only)."""
import numpy as np
import pytest
from sklearn.covariance import ledoit_wolf

from oracle.calib import (FLOOR_REL, calib_precond, channel_moments, diag_preconditioner,
                          ledoit_wolf_diag)


def test_constant_magnitude_channels_give_exact_moments_and_no_shrinkage():
    # |x_tj| = c_j for every token: s = c^2, q = c^4, so beta_bar = 0 and alpha = 0.
    rng = np.random.default_rng(0)
    c = np.array([0.5, 1.0, 2.0, 3.0])
    x = c[None, :] * np.where(rng.random((1000, 4)) < 0.5, -1.0, 1.0)
    s, q, T = channel_moments([x])
    np.testing.assert_allclose(s, c ** 2, rtol=0, atol=1e-15)
    np.testing.assert_allclose(q, c ** 4, rtol=1e-15)
    alpha, dtilde, _ = ledoit_wolf_diag(s, q, T)
    assert alpha == 0.0
    np.testing.assert_allclose(dtilde, c ** 2)
    d, _ = diag_preconditioner(s, q, T)
    np.testing.assert_allclose(d, c, rtol=1e-15)


def test_equal_channels_mean_no_dispersion():
    # all second moments equal: delta^2 = 0, alpha = 1 by convention, and d~ = s = mu.
    x = np.ones((8, 5)) * np.array([1, -1, 1, -1, 1])[None, :]
    x[::2] *= 2.0
    s, q, T = channel_moments([x])
    alpha, dtilde, mu = ledoit_wolf_diag(s, q, T)
    assert alpha == 1.0
    np.testing.assert_allclose(dtilde, s)


def test_chunking_does_not_change_moments():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((1000, 7)) * np.exp(rng.standard_normal(7))
    s1, q1, T1 = channel_moments([x])
    s2, q2, T2 = channel_moments([x[:333], x[333:334], x[334:]])
    assert T1 == T2 == 1000
    np.testing.assert_allclose(s1, s2, rtol=1e-14)
    np.testing.assert_allclose(q1, q2, rtol=1e-14)
    np.testing.assert_allclose(s1, (x ** 2).mean(0), rtol=1e-14)
    np.testing.assert_allclose(q1, (x ** 4).mean(0), rtol=1e-14)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_one_hot_tokens_match_sklearn_full_ledoit_wolf(seed):
    # When every token activates one channel, the sample second-moment matrix and every
    # per-token outer product are diagonal, so the full-matrix LW-2004 estimator reduces
    # exactly to the diagonal restriction.  sklearn implements the full estimator.
    rng = np.random.default_rng(seed)
    T, p = 400, 6
    ch = rng.integers(0, p, size=T)
    val = rng.standard_normal(T) * np.exp(rng.standard_normal(p))[ch]
    X = np.zeros((T, p))
    X[np.arange(T), ch] = val
    s, q, TT = channel_moments([X])
    alpha, dtilde, _ = ledoit_wolf_diag(s, q, TT)
    shrunk, shrinkage = ledoit_wolf(X, assume_centered=True)
    assert abs(alpha - shrinkage) < 1e-12
    np.testing.assert_allclose(dtilde, np.diag(shrunk), rtol=1e-12)
    assert 0.0 < alpha <= 1.0


def test_alpha_in_unit_interval_and_decreases_with_tokens():
    rng = np.random.default_rng(3)
    scales = np.exp(rng.standard_normal(64))
    alphas = []
    for T in [64, 1024, 16384]:
        x = rng.standard_normal((T, 64)) * scales
        s, q, TT = channel_moments([x])
        a, _, _ = ledoit_wolf_diag(s, q, TT)
        assert 0.0 <= a <= 1.0
        alphas.append(a)
    assert alphas[0] > alphas[1] > alphas[2]


def test_zero_channel_is_floored_and_override_applies():
    x = np.zeros((10, 3))
    x[:, 0] = 1.0
    x[:, 1] = -2.0
    s, q, T = channel_moments([x])
    d, a = diag_preconditioner(s, q, T)
    _, dtilde, mu = ledoit_wolf_diag(s, q, T)
    assert d[2] >= np.sqrt(FLOOR_REL * mu) * (1 - 1e-12)
    d_fixed, a_fixed = diag_preconditioner(s, q, T, alpha_override=0.25)
    assert a_fixed == 0.25
    np.testing.assert_allclose(d_fixed ** 2, np.maximum(0.75 * s + 0.25 * s.mean(), FLOOR_REL * s.mean()))


def test_calib_precond_pairs_streams_with_sides():
    rng = np.random.default_rng(4)
    acts = rng.standard_normal((100, 5))
    grads = 3.0 * rng.standard_normal((100, 2))
    d_in, d_out, a_in, a_out = calib_precond([acts], [grads])
    assert d_in.shape == (5,) and d_out.shape == (2,)
    assert np.all(d_out > 2.0) and np.all(d_in < 2.0)
