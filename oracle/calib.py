"""Calibration statistics and Ledoit-Wolf diagonal preconditioners (oracle side).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

Passages followed (NanoQuant summary page, paper.rainbus.top):
  * "Method steps" (方法步骤详情), stage one (global calibration): a forward pass
    over 128 calibration sequences of 2048 tokens collects, for every linear
    layer, the statistics z_in and z_out, which Ledoit-Wolf shrinkage turns into
    robust diagonal preconditioners D_in and D_out.
  * "Prerequisites" (前置知识), K-FAC paragraph: the Hessian is approximated by
    Kronecker factors simplified to their diagonals.

Readings where the pages are silent:
  * z_in are the uncentred second moments of the layer's input activations
    (length n), z_out those of the gradients at the layer's output (length m),
    i.e. the diagonals of the K-FAC factors E[x x^T] and E[g g^T].
  * Ledoit-Wolf is the 2004 estimator (Ledoit & Wolf, J. Multivariate Anal. 88)
    with target mu.I, restricted to the diagonal of the sample second-moment
    matrix: the only part a per-channel reduction produces.
  * D = diag(sqrt(d~)), so that ||D_out (W - W') D_in||_F^2 is the diagonal K-FAC
    quadratic form sum_ij G_ii A_jj (W - W')_ij^2.
  * Channels whose shrunk moment is below 1e-12 * mu are floored there.
"""
import numpy as np

FLOOR_REL = 1e-12


def channel_moments(chunks):
    """Per-channel s_j = mean_t x_tj^2 and q_j = mean_t x_tj^4 over a token stream.

    ``chunks`` is an iterable of (T_i x C) arrays (any float dtype); they are
    promoted to float64 one chunk at a time so that long streams fit in memory.
    Returns (s, q, T).
    """
    s = None
    q = None
    T = 0
    for x in chunks:
        x = np.asarray(x, dtype=np.float64)
        if x.ndim != 2:
            raise ValueError("stream chunks must be 2-D (tokens x channels)")
        x2 = x * x
        if s is None:
            s = np.zeros(x.shape[1])
            q = np.zeros(x.shape[1])
        s += x2.sum(axis=0)
        q += (x2 * x2).sum(axis=0)
        T += x.shape[0]
    if T == 0:
        raise ValueError("empty calibration stream")
    return s / T, q / T, T


def ledoit_wolf_diag(s, q, T):
    """Shrinkage intensity alpha and shrunk diagonal d~ of the sample moment matrix.

    With p channels, S the sample second-moment matrix (diagonal part s) and
    target mu.I, mu = mean(s):
        delta^2 = sum_j (s_j - mu)^2                    (dispersion of S about the target)
        beta_bar^2 = (1/T) sum_j (q_j - s_j^2)          (variance of the per-token terms)
        beta^2 = min(beta_bar^2, delta^2)
        alpha = beta^2 / delta^2   (1 when delta^2 = 0)
        d~ = (1 - alpha) s + alpha mu
    The common 1/p normalisation of the Frobenius norms cancels in alpha.
    """
    s = np.asarray(s, dtype=np.float64)
    q = np.asarray(q, dtype=np.float64)
    mu = s.mean()
    delta2 = float(((s - mu) ** 2).sum())
    beta_bar2 = float((q - s * s).sum()) / T
    beta2 = min(beta_bar2, delta2)
    alpha = 1.0 if delta2 == 0.0 else beta2 / delta2
    dtilde = (1.0 - alpha) * s + alpha * mu
    return alpha, dtilde, mu


def diag_preconditioner(s, q, T, alpha_override=None):
    """d = sqrt(max(d~, 1e-12 mu)) with d~ from Ledoit-Wolf (or a fixed alpha).

    Returns (d, alpha).
    """
    alpha, dtilde, mu = ledoit_wolf_diag(s, q, T)
    if alpha_override is not None and alpha_override >= 0.0:
        alpha = float(alpha_override)
        dtilde = (1.0 - alpha) * np.asarray(s, dtype=np.float64) + alpha * mu
    dtilde = np.maximum(dtilde, FLOOR_REL * mu)
    return np.sqrt(dtilde), alpha


def calib_precond(act_chunks, grad_chunks, alpha_override=None):
    """Stage-one preconditioners: d_in from the activation stream, d_out from the gradients."""
    s_in, q_in, T_in = channel_moments(act_chunks)
    s_out, q_out, T_out = channel_moments(grad_chunks)
    d_in, a_in = diag_preconditioner(s_in, q_in, T_in, alpha_override)
    d_out, a_out = diag_preconditioner(s_out, q_out, T_out, alpha_override)
    return d_in, d_out, a_in, a_out
