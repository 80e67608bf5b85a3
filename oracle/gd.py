"""Gradient-descent latent update (the community page's solver variant), FP64 oracle.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

Passage followed: community blog page (bittide.aicompass.dev), to-do section (待办事项):
the implementer replaced LB-ADMM's Cholesky solves of the linear systems by a
gradient-descent solver, slower than Cholesky on CUDA and faster on an Intel Arc B580.
The page gives neither a step rule nor a step count; this module takes the plainest
reading:
  * the U-step minimises f(X) = 1/2 ||A - X Y^T||^2 + lam/2 ||X||^2 + rho/2 ||X - Z + L||^2,
    whose gradient is X G - R with G = Y^T Y + (lam + rho) I and R = A Y + rho (Z - L);
  * a step is X <- X - eta (X G - R) with eta = 1 / ||G||_inf (the largest absolute row
    sum of G, an upper bound of its largest eigenvalue, so that no step increases f);
  * each half iteration starts from the side's current latent (zero for U before the
    first U-step) and takes ``steps`` steps; the rest of LB-ADMM is unchanged.
"""
import numpy as np

from . import lbadmm as O


def gd_step_size(G):
    """eta = 1 / max_i sum_j |G_ij|."""
    return 1.0 / float(np.max(np.sum(np.abs(G), axis=1)))


def latent_objective(A, X, Y, Z, Lam, rho, lam):
    """f(X) written out from its definition (not from the gradient)."""
    D = A - X @ Y.T
    E = X - Z + Lam
    return 0.5 * float(np.sum(D * D)) + 0.5 * lam * float(np.sum(X * X)) + \
        0.5 * rho * float(np.sum(E * E))


def latent_update_gd(A, Y, Z, Lam, X0, rho, lam, steps):
    """``steps`` gradient steps from X0.  Returns (X, G, R, eta)."""
    A = np.asarray(A, dtype=np.float64)
    Y = np.asarray(Y, dtype=np.float64)
    r = Y.shape[1]
    G = Y.T @ Y + (lam + rho) * np.eye(r)
    R = A @ Y + rho * (np.asarray(Z, dtype=np.float64) - np.asarray(Lam, dtype=np.float64))
    eta = gd_step_size(G)
    X = np.asarray(X0, dtype=np.float64).copy()
    for _ in range(steps):
        X = X - eta * (X @ G - R)
    return X, G, R, eta


def lbadmm_gd(W, d_in=None, d_out=None, r=16, rho=1.0, lam=1e-4, iters=30, K=4, seed=0,
              steps=8):
    """LB-ADMM with the gradient-descent latent updates; everything else as oracle.lbadmm
    (same order, SVID, dual update, objective, balancing, scales, packing)."""
    Wt, What, gamma = O.precondition(W, d_in, d_out, r)
    m, n = What.shape
    V = O.init_latent(n, r, seed)
    U = np.zeros((m, r))
    ZU, LU = np.zeros((m, r)), np.zeros((m, r))
    ZV, LV = np.zeros((n, r)), np.zeros((n, r))
    objective = []
    for _ in range(iters):
        U, _, _, _ = latent_update_gd(What, V, ZU, LU, U, rho, lam, steps)
        ZU, _, _ = O.svid(U + LU, K)
        LU = O.dual_update(LU, U, ZU)
        V, _, _, _ = latent_update_gd(What.T, U, ZV, LV, V, rho, lam, steps)
        ZV, _, _ = O.svid(V + LV, K)
        LV = O.dual_update(LV, V, ZV)
        objective.append(O.relative_residual(What, U, V))
    Ub, Vb, _ = O.balance(U, V)
    s1, s2 = O.extract_scales(Ub, Vb, gamma)
    err = O.recon_error(Wt, s1, O.sign_pm(Ub), O.sign_pm(Vb), s2)
    return O.LBADMMResult(O.pack_signs(Ub), O.pack_signs(Vb), s1, s2, objective, err, gamma,
                          Ub, Vb, [])
