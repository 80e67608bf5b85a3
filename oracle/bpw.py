"""Bits-per-weight accounting and per-layer rank selection (oracle side).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

The representation is W ~ diag(s1) . U+-1 . V+-1^T . diag(s2) with U (m x r) and
V (n x r) in {+1,-1} (NanoQuant summary page, "Motivation" (研究动机), the
low-rank binary form s1.U.V^T.s2; "Prerequisites" (前置知识), low-rank
factorisation paragraph).  Storing it costs one bit per sign, (m+n).r bits, plus
the two scale vectors, which are kept at 16 bits each: 16.(m+n) bits.  Dividing
by the m.n weights gives the bits per weight (BPW) the pages quote (1.00, 0.80,
0.55 BPW in the results section, 实验结果).  Exact rational arithmetic is used so
that the floor in ``rank_for_bpw`` is never off by one.
"""
from fractions import Fraction
import math


def _exact(x):
    """Exact rational value of a decimal literal such as 0.55 (not its binary double)."""
    if isinstance(x, Fraction):
        return x
    if isinstance(x, int):
        return Fraction(x)
    return Fraction(repr(float(x)))


def bpw(m, n, r):
    """BPW of an m x n layer stored as rank-r binary factors plus 16-bit scales.

    ((m+n).r + 16.(m+n)) / (m.n), returned as an exact Fraction.
    """
    m, n, r = int(m), int(n), int(r)
    if m <= 0 or n <= 0 or r < 0:
        raise ValueError("m, n must be positive and r non-negative")
    return Fraction((m + n) * r + 16 * (m + n), m * n)


def rank_for_bpw(m, n, target):
    """Largest rank whose BPW does not exceed ``target`` (uniform-BPW rank choice).

    r = floor((target.m.n - 16.(m+n)) / (m+n)), clamped at 0.  The pages give a
    single rank parameter per model (limitations section, 局限与改进); per-layer
    BPW targets are met by taking this floor for each layer's shape.
    """
    m, n = int(m), int(n)
    t = _exact(target)
    r = math.floor((t * m * n - 16 * (m + n)) / (m + n))
    return max(int(r), 0)


def linear_bits(layers, target):
    """Total bits of a list of (m, n) linear layers, each at its own floor rank."""
    total = 0
    for m, n in layers:
        r = rank_for_bpw(m, n, target)
        total += (m + n) * r + 16 * (m + n)
    return total


def nominal_linear_bits(layers, target):
    """Bits of the same layers if every layer sat exactly at ``target`` BPW."""
    t = _exact(target)
    return sum(t * m * n for m, n in layers)
