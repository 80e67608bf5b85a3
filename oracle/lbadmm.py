"""Latent Binary ADMM (LB-ADMM) initialisation, FP64 oracle.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

Passages followed (NanoQuant summary page, paper.rainbus.top):
  * "Motivation" (研究动机): the target form W ~ s1 . U+-1 . V+-1^T . s2.
  * "Core method" (核心方法): continuous latents U, V relax the binary factors;
    each iteration (a) fixes V and solves U's regularised linear system by a
    Cholesky factorisation, (b) maps U to a binary proxy Z with SVID
    (Sign-Value Independent Decomposition), (c) updates the dual variable to
    enforce consistency; the V side mirrors it.
  * "Method steps" (方法步骤详情), stage two: the preconditioned target
    W~ = D_out . W . D_in; after convergence magnitude balancing removes the
    scale ambiguity, the channel scales s1 and s2 are extracted, and the signs are
    packed into integers.
  * "Technical novelty" (技术新颖性): SVID handles the discrete proxy update;
    magnitude balancing removes the low-rank scale ambiguity.

The pages print no equations.  This module takes the following concrete form,
stated once here and restated where used:
  * U-step  U <- (W^ V + rho (Z_U - L_U)) (V^T V + (lambda + rho) I)^-1, i.e. the
    exact minimiser over U of
        1/2 ||W^ - U V^T||^2 + lambda/2 ||U||^2 + rho/2 ||U - Z_U + L_U||^2,
    solved with a Cholesky factor of the r x r system matrix.
  * SVID    S = U + L_U, A = |S|, b = 1_r, K times {a = A b / ||A b||, b = A^T a},
    Z_U = sign(S) * a b^T  (rank-1 fit of |S| by K power steps).
  * dual    L_U <- L_U + U - Z_U.
  * V-step  the same with W^^T and U.
  * W^ = W~ / gamma with gamma = ||W~||_F / (2 sqrt(r)), i.e. ||W^||_F = 2 sqrt(r):
    the singular values of the rank-r part of W^ are then of order 2, so that
    rho = 1 weighs the consensus term at about half the curvature V^T V of the
    data term, whatever the layer's size and scale.  gamma is folded back into s1.
  * V_0 = sqrt(2/n) . (+-1 signs from SplitMix64(seed)), whose Gram is close to
    2 I (the balanced scale of the normalised target); Z and L start at 0.
  * Balancing equalises ||U_:k|| and ||V_:k|| per rank column; s1 and s2 are the
    row mean-abs values of the balanced latents (s1 times gamma); a sign bit is 1
    exactly where the balanced latent is < 0 (so -0.0 and 0 map to +1).
  * Packing: LSB-first along the rank index, row-major uint32[rows][ceil(r/32)],
    padding bits 0.
"""
from dataclasses import dataclass, field
from typing import List, Optional

import numpy as np
from scipy.linalg import cho_factor, cho_solve

from .splitmix import sign_matrix

NORMAL_EQ_TOL = 1e-10


class NormalEquationError(AssertionError):
    pass


def precondition(W, d_in=None, d_out=None, r=1):
    """W~ = diag(d_out) W diag(d_in), gamma = ||W~||_F / (2 sqrt(r)), W^ = W~ / gamma.

    Returns (W~, W^, gamma).  A zero W~ gives gamma = 0 and W^ = 0.
    """
    W = np.asarray(W, dtype=np.float64)
    m, n = W.shape
    d_in = np.ones(n) if d_in is None else np.asarray(d_in, dtype=np.float64)
    d_out = np.ones(m) if d_out is None else np.asarray(d_out, dtype=np.float64)
    Wt = d_out[:, None] * W * d_in[None, :]
    gamma = float(np.linalg.norm(Wt)) / (2.0 * np.sqrt(r))
    What = Wt / gamma if gamma > 0.0 else np.zeros_like(Wt)
    return Wt, What, gamma


def init_latent(rows, r, seed):
    """V_0[j, k] = sqrt(2 / rows) * sign drawn from SplitMix64(seed, j*r + k)."""
    return np.sqrt(2.0 / rows) * sign_matrix(seed, rows, r)


def latent_update(A, Y, Z, Lam, rho, lam, check=True):
    """X = (A Y + rho (Z - Lam)) (Y^T Y + (lam + rho) I)^-1 by Cholesky.

    This is the minimiser over X of
        1/2 ||A - X Y^T||_F^2 + lam/2 ||X||_F^2 + rho/2 ||X - Z + Lam||_F^2
    (stationarity: -(A - X Y^T) Y + lam X + rho (X - Z + Lam) = 0).
    Returns (X, G, R, residual) with residual = ||X G - R||_F / ||R||_F, which
    must stay below 1e-10 when ``check`` is set.
    """
    r = Y.shape[1]
    G = Y.T @ Y + (lam + rho) * np.eye(r)
    R = A @ Y + rho * (Z - Lam)
    factor = cho_factor(G, lower=True)
    X = cho_solve(factor, R.T).T
    nR = float(np.linalg.norm(R))
    resid = float(np.linalg.norm(X @ G - R)) / nR if nR > 0.0 else 0.0
    if check and not resid < NORMAL_EQ_TOL:
        raise NormalEquationError(f"normal-equation residual {resid:.3e} >= {NORMAL_EQ_TOL}")
    return X, G, R, resid


def sign_pm(S):
    """+1 where S >= 0 (including -0.0), -1 where S < 0."""
    return np.where(S < 0, -1.0, 1.0)


def svid(S, K):
    """Sign-Value Independent Decomposition: Z = sign(S) * a b^T.

    a b^T is the rank-1 fit of A = |S| reached by K power steps started from
    b = 1: a = A b / ||A b||, b = A^T a.  If A b vanishes, a = b = 0 (Z = 0).
    Returns (Z, a, b).
    """
    if K < 1:
        raise ValueError("SVID needs at least one power step")
    A = np.abs(S)
    rows, r = A.shape
    a = np.zeros(rows)
    b = np.ones(r)
    for _ in range(K):
        t = A @ b
        nt = float(np.linalg.norm(t))
        if nt == 0.0:
            a = np.zeros(rows)
            b = np.zeros(r)
            break
        a = t / nt
        b = A.T @ a
    Z = sign_pm(S) * np.outer(a, b)
    return Z, a, b


def dual_update(Lam, X, Z):
    """L <- L + X - Z."""
    return Lam + X - Z


def relative_residual(What, U, V):
    """||W^ - U V^T||_F^2 / ||W^||_F^2 (0 for a zero target)."""
    n2 = float(np.sum(What * What))
    if n2 == 0.0:
        return 0.0
    D = What - U @ V.T
    return float(np.sum(D * D)) / n2


def balance(U, V):
    """Per rank column k: U_:k *= g_k, V_:k /= g_k with g_k = sqrt(||V_:k|| / ||U_:k||).

    After this ||U_:k|| = ||V_:k|| and U V^T is unchanged.  g_k = 1 when either
    norm is zero.
    """
    nu = np.linalg.norm(U, axis=0)
    nv = np.linalg.norm(V, axis=0)
    g = np.ones(U.shape[1])
    ok = (nu > 0) & (nv > 0)
    g[ok] = np.sqrt(nv[ok] / nu[ok])
    return U * g[None, :], V / g[None, :], g


def extract_scales(Ub, Vb, gamma):
    """s1_i = gamma * mean_k |U_ik|, s2_j = mean_k |V_jk| (least-squares scale of sign(x) for x)."""
    return gamma * np.abs(Ub).mean(axis=1), np.abs(Vb).mean(axis=1)


def pack_signs(X):
    """uint32[rows][ceil(r/32)]: bit (k mod 32) of word k//32 is 1 iff X[:, k] < 0."""
    X = np.asarray(X)
    rows, r = X.shape
    words = (r + 31) // 32
    out = np.zeros((rows, words), dtype=np.uint64)
    neg = (X < 0)
    for k in range(r):
        out[:, k // 32] |= neg[:, k].astype(np.uint64) << np.uint64(k % 32)
    return out.astype(np.uint32)


def unpack_signs(P, r):
    """Inverse of ``pack_signs``: rows x r matrix of +-1."""
    P = np.asarray(P, dtype=np.uint64)
    rows = P.shape[0]
    out = np.ones((rows, r))
    for k in range(r):
        bit = (P[:, k // 32] >> np.uint64(k % 32)) & np.uint64(1)
        out[bit == 1, k] = -1.0
    return out


def reconstruct(s1, Us, Vs, s2):
    """diag(s1) U+- V+-^T diag(s2)."""
    return (np.asarray(s1)[:, None] * (Us @ Vs.T)) * np.asarray(s2)[None, :]


def recon_error(Wt, s1, Us, Vs, s2):
    """||W~ - diag(s1) U+- V+-^T diag(s2)||_F / ||W~||_F (0 when both vanish)."""
    D = Wt - reconstruct(s1, Us, Vs, s2)
    nd = float(np.linalg.norm(D))
    nw = float(np.linalg.norm(Wt))
    if nw == 0.0:
        return 0.0 if nd == 0.0 else float("inf")
    return nd / nw


@dataclass
class LBADMMResult:
    U_packed: np.ndarray
    V_packed: np.ndarray
    s1: np.ndarray
    s2: np.ndarray
    objective: List[float]
    rel_err: float
    gamma: float
    U: np.ndarray            # balanced latents (m x r)
    V: np.ndarray            # balanced latents (n x r)
    residuals: List[float] = field(default_factory=list)


def lbadmm(W, d_in=None, d_out=None, r=16, rho=1.0, lam=1e-4, iters=30, K=4, seed=0,
           V0=None, check=True, on_iter=None):
    """Full LB-ADMM initialisation of one layer.

    Order per iteration: U-step, SVID(U), dual(U); V-step, SVID(V), dual(V);
    objective ||W^ - U V^T||^2 / ||W^||^2.  After ``iters`` iterations the last
    latents are balanced, the scales extracted, the signs packed and the
    reconstruction error of the packed form against W~ returned.
    ``on_iter(t, state_dict)`` is called after every iteration when given.
    """
    if r < 1:
        raise ValueError("rank must be >= 1")
    Wt, What, gamma = precondition(W, d_in, d_out, r)
    m, n = What.shape
    V = init_latent(n, r, seed) if V0 is None else np.asarray(V0, dtype=np.float64).copy()
    U = np.zeros((m, r))
    ZU = np.zeros((m, r))
    LU = np.zeros((m, r))
    ZV = np.zeros((n, r))
    LV = np.zeros((n, r))
    objective = []
    residuals = []
    for t in range(iters):
        U, _, _, ru = latent_update(What, V, ZU, LU, rho, lam, check)
        ZU, _, _ = svid(U + LU, K)
        LU = dual_update(LU, U, ZU)
        V, _, _, rv = latent_update(What.T, U, ZV, LV, rho, lam, check)
        ZV, _, _ = svid(V + LV, K)
        LV = dual_update(LV, V, ZV)
        residuals.extend([ru, rv])
        objective.append(relative_residual(What, U, V))
        if on_iter is not None:
            on_iter(t, dict(U=U, V=V, ZU=ZU, LU=LU, ZV=ZV, LV=LV))
    Ub, Vb, _ = balance(U, V)
    s1, s2 = extract_scales(Ub, Vb, gamma)
    Us = sign_pm(Ub)
    Vs = sign_pm(Vb)
    err = recon_error(Wt, s1, Us, Vs, s2)
    return LBADMMResult(pack_signs(Ub), pack_signs(Vb), s1, s2, objective, err, gamma,
                        Ub, Vb, residuals)
