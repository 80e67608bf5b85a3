"""Counter-based SplitMix64 generator (oracle side).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

The pages name a seed but no initialisation for the ADMM latents.  The reading
used here draws the initial signs of V from SplitMix64 (Steele, Lea and Flood,
"Fast splittable pseudorandom number generators", OOPSLA 2014; the public-domain
reference ``splitmix64.c`` by S. Vigna), evaluated as a pure function of a
counter so that any element can be produced independently:

    z = seed + (idx + 1) * 0x9E3779B97F4A7C15          (mod 2^64)
    z = (z xor (z >> 30)) * 0xBF58476D1CE4E5B9
    z = (z xor (z >> 27)) * 0x94D049BB133111EB
    out = z xor (z >> 31)

``out`` equals the (idx+1)-th output of the sequential generator started at
state ``seed``.  The CUDA side has its own implementation of the same published
definition; the two share no code.
"""
import numpy as np

_MASK = (1 << 64) - 1
_GOLDEN = 0x9E3779B97F4A7C15
_MUL1 = 0xBF58476D1CE4E5B9
_MUL2 = 0x94D049BB133111EB


def splitmix64_scalar(seed, idx):
    """One output as a Python int, computed with unbounded integers then masked."""
    z = (int(seed) + (int(idx) + 1) * _GOLDEN) & _MASK
    z = ((z ^ (z >> 30)) * _MUL1) & _MASK
    z = ((z ^ (z >> 27)) * _MUL2) & _MASK
    return z ^ (z >> 31)


def splitmix64(seed, idx):
    """Vectorised outputs for an array of counters (uint64 wrap-around arithmetic)."""
    idx = np.asarray(idx, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(int(seed) & _MASK) + (idx + np.uint64(1)) * np.uint64(_GOLDEN)
        z = (z ^ (z >> np.uint64(30))) * np.uint64(_MUL1)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(_MUL2)
        z = z ^ (z >> np.uint64(31))
    return z


def sign_matrix(seed, rows, cols):
    """rows x cols matrix of +-1: -1 where the top bit of splitmix64(seed, i*cols+k) is set."""
    idx = np.arange(rows * cols, dtype=np.uint64)
    top = splitmix64(seed, idx) >> np.uint64(63)
    return np.where(top == 1, -1.0, 1.0).reshape(rows, cols)
