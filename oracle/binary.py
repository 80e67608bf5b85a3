"""Inference with the packed binary factors, FP64 oracle.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

Passage followed: NanoQuant summary page (paper.rainbus.top), "Technical novelty"
(技术新颖性) and "Limitations" (局限与改进): the compressed layer is applied through custom
binary GEMV/GEMM kernels that work on the packed signs, y = W_q x with
W_q = diag(s1) U+- V+-^T diag(s2).  For a batch of B input rows X (B x n):

    Y = X diag(s2) V+- U+-^T diag(s1)          (B x m)

computed here in the plain order: unpack the signs, form the two skinny products.
"""
import numpy as np

from .lbadmm import unpack_signs


def binary_matmul(X, U_packed, V_packed, s1, s2, r):
    """Y[b, i] = s1_i sum_k U+-[i, k] sum_j V+-[j, k] s2_j X[b, j], in FP64."""
    X = np.atleast_2d(np.asarray(X, dtype=np.float64))
    Us = unpack_signs(U_packed, r)
    Vs = unpack_signs(V_packed, r)
    Z = (X * np.asarray(s2, dtype=np.float64)[None, :]) @ Vs      # B x r
    return (Z @ Us.T) * np.asarray(s1, dtype=np.float64)[None, :]  # B x m


def binary_matmul_loops(X, U_packed, V_packed, s1, s2, r):
    """The same by explicit loops over the packed words (tiny inputs only)."""
    X = np.atleast_2d(np.asarray(X, dtype=np.float64))
    B, n = X.shape
    m = len(s1)
    U_packed = np.asarray(U_packed, dtype=np.uint64)
    V_packed = np.asarray(V_packed, dtype=np.uint64)
    Y = np.zeros((B, m))
    for b in range(B):
        z = [0.0] * r
        for j in range(n):
            w = float(s2[j]) * float(X[b, j])
            for k in range(r):
                neg = (int(V_packed[j, k // 32]) >> (k % 32)) & 1
                z[k] += -w if neg else w
        for i in range(m):
            acc = 0.0
            for k in range(r):
                neg = (int(U_packed[i, k // 32]) >> (k % 32)) & 1
                acc += -z[k] if neg else z[k]
            Y[b, i] = float(s1[i]) * acc
    return Y
