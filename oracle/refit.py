"""Least-squares refit of the channel scales with the signs fixed, FP64 oracle.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

Passages followed (NanoQuant summary page, paper.rainbus.top): "Method steps" (方法步骤详情),
stage two, and "Technical novelty" (技术新颖性): after the ADMM the scale ambiguity of the
factors is removed (magnitude balancing) and the channel-wise scales s1, s2 of
W~ ~ diag(s1) U+- V+-^T diag(s2) are extracted.  The extraction from the balanced latents
(row mean-abs values) is not the least-squares optimum of those scales for the fixed
signs; this module refines them by alternating exact minimisations with the signs held:

    P = U+- V+-^T                                    (integers in [-r, r])
    s1_i <- sum_j W~_ij P_ij s2_j / sum_j P_ij^2 s2_j^2      (s2 fixed)
    s2_j <- sum_i W~_ij P_ij s1_i / sum_i P_ij^2 s1_i^2      (s1 fixed)

A scale whose denominator vanishes keeps its value.  Each half sweep is the exact
minimiser of the squared error over one block of scales, so the error never increases.
"""
import numpy as np


def ls_refit(Wt, Us, Vs, s1, s2, sweeps=3):
    """Returns (s1, s2, errors) with errors[k] = ||W~ - diag(s1) P diag(s2)||_F / ||W~||_F
    after k sweeps (errors[0]: the starting scales)."""
    Wt = np.asarray(Wt, dtype=np.float64)
    P = np.asarray(Us, dtype=np.float64) @ np.asarray(Vs, dtype=np.float64).T
    s1 = np.asarray(s1, dtype=np.float64).copy()
    s2 = np.asarray(s2, dtype=np.float64).copy()
    nw = float(np.linalg.norm(Wt))

    def err():
        d = Wt - (s1[:, None] * P) * s2[None, :]
        return float(np.linalg.norm(d)) / nw if nw > 0 else 0.0

    errors = [err()]
    for _ in range(sweeps):
        num = (Wt * P) @ s2
        den = (P * P) @ (s2 * s2)
        ok = den > 0
        s1[ok] = num[ok] / den[ok]
        num = (Wt * P).T @ s1
        den = (P * P).T @ (s1 * s1)
        ok = den > 0
        s2[ok] = num[ok] / den[ok]
        errors.append(err())
    return s1, s2, errors
