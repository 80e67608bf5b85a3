"""Pins for the oracle's SplitMix64 generator (CPU only)."""
import numpy as np

from conftest import read_golden
from oracle.splitmix import sign_matrix, splitmix64, splitmix64_scalar


def test_published_test_vector():
    for seed, idx, out in read_golden("splitmix64.txt"):
        assert splitmix64_scalar(int(seed), int(idx)) == int(out)
        assert int(splitmix64(int(seed), [int(idx)])[0]) == int(out)


def test_vectorised_matches_scalar_for_large_seeds():
    seed = (1 << 64) - 12345
    idx = np.array([0, 1, 2, 1000, (1 << 40) + 7], dtype=np.uint64)
    got = splitmix64(seed, idx)
    for i, v in zip(idx, got):
        assert int(v) == splitmix64_scalar(seed, int(i))


def test_sign_matrix_uses_top_bit_row_major():
    M = sign_matrix(7, 3, 5)
    for i in range(3):
        for k in range(5):
            top = splitmix64_scalar(7, i * 5 + k) >> 63
            assert M[i, k] == (-1.0 if top else 1.0)
    big = sign_matrix(0, 256, 64)
    assert abs(big.mean()) < 0.02      # balanced signs
