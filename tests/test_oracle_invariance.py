"""Exact invariances of the oracle that follow from the method's definitions.

* Scaling W by c scales W~ and gamma = ||W~||_F / (2 sqrt r) by c and leaves W^ = W~/gamma
  unchanged, so the iteration, the signs and s2 are unchanged, s1 (which carries gamma)
  scales by c, and the relative reconstruction error is unchanged.  With c a power of two
  every step is exact in floating point, so the comparison is bitwise.
* The preconditioners enter only through W~ = D_out W D_in.
* Scaling a calibration stream by c scales the second moments by c^2 and the fourth by
  c^4: the Ledoit-Wolf intensity (a ratio of quantities of degree 4) is unchanged and
  d = sqrt(d~) scales by |c|.  Permuting channels permutes d.
"""
import numpy as np
import pytest

from oracle import calib as OC
from oracle import lbadmm as O


def _layer(seed, m=40, n=56):
    rng = np.random.default_rng(seed)
    return rng.standard_normal((m, n)) * np.exp(0.5 * rng.standard_normal(n))[None, :]


def test_weight_scale_power_of_two_is_bitwise_invariant():
    W = _layer(1)
    a = O.lbadmm(W, r=6, iters=8)
    b = O.lbadmm(32.0 * W, r=6, iters=8)
    np.testing.assert_array_equal(a.U_packed, b.U_packed)
    np.testing.assert_array_equal(a.V_packed, b.V_packed)
    np.testing.assert_array_equal(a.s2, b.s2)
    np.testing.assert_array_equal(32.0 * a.s1, b.s1)
    assert a.rel_err == b.rel_err and a.objective == b.objective


def test_weight_scale_general_is_invariant_to_rounding():
    W = _layer(2)
    a = O.lbadmm(W, r=5, iters=6)
    b = O.lbadmm(3.7 * W, r=5, iters=6)
    np.testing.assert_array_equal(a.U_packed, b.U_packed)
    np.testing.assert_array_equal(a.V_packed, b.V_packed)
    np.testing.assert_allclose(b.s1, 3.7 * a.s1, rtol=1e-9)
    np.testing.assert_allclose(b.s2, a.s2, rtol=1e-9)
    assert abs(a.rel_err - b.rel_err) <= 1e-9 * a.rel_err


def test_preconditioners_enter_only_through_the_scaled_weight():
    W = _layer(3, 36, 48)
    rng = np.random.default_rng(4)
    d_in = np.exp(rng.standard_normal(48))
    d_out = np.exp(rng.standard_normal(36))
    a = O.lbadmm(W, d_in, d_out, r=4, iters=6)
    Wt = d_out[:, None] * W * d_in[None, :]
    b = O.lbadmm(Wt, np.ones(48), np.ones(36), r=4, iters=6)
    np.testing.assert_array_equal(a.U_packed, b.U_packed)
    np.testing.assert_array_equal(a.V_packed, b.V_packed)
    np.testing.assert_array_equal(a.s1, b.s1)
    np.testing.assert_array_equal(a.s2, b.s2)
    assert a.rel_err == b.rel_err


def _stream(seed, T, C):
    rng = np.random.default_rng(seed)
    return rng.standard_normal((T, C)) * np.exp(rng.standard_normal(C))[None, :]


@pytest.mark.parametrize("c", [4.0, -0.5, 3.0])
def test_stream_scale_covariance(c):
    X, G = _stream(5, 512, 24), _stream(6, 384, 16)
    d_in, d_out, a_in, a_out = OC.calib_precond([X], [G])
    e_in, e_out, b_in, b_out = OC.calib_precond([c * X], [c * G])
    exact = c in (4.0, -0.5)
    rtol = 0.0 if exact else 1e-12
    np.testing.assert_allclose(e_in, abs(c) * d_in, rtol=rtol, atol=0)
    np.testing.assert_allclose(e_out, abs(c) * d_out, rtol=rtol, atol=0)
    assert abs(b_in - a_in) <= (0.0 if exact else 1e-12) and abs(b_out - a_out) <= (
        0.0 if exact else 1e-12)


def test_channel_permutation_equivariance():
    X, G = _stream(7, 640, 30), _stream(8, 640, 20)
    perm = np.random.default_rng(9).permutation(30)
    d_in, _, a_in, _ = OC.calib_precond([X], [G])
    p_in, _, b_in, _ = OC.calib_precond([X[:, perm]], [G])
    np.testing.assert_allclose(p_in, d_in[perm], rtol=1e-12)
    assert abs(a_in - b_in) <= 1e-12
