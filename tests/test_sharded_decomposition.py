"""Row-sharded LB-ADMM of one layer: the exchange steps, checked on CPU with gloo ranks.

Sharding one m x n layer by rows over ranks k (W~_k: rows of rank k) keeps the U side
local and replicates V.  The exchanges one iteration needs are exactly:
  * gamma:   ||W~||^2 = sum_k ||W~_k||^2                     (once, one scalar)
  * U step:  none - G_V = V^T V + (lambda + rho) I is formed from the replicated V;
             U_k = (W^_k V + rho (Z_U,k - L_U,k)) G_V^-1 on the rank's rows
  * SVID(U): per power step ||t||^2 = sum_k ||t_k||^2 (one scalar) and
             b = sum_k |S_k|^T a_k (r values)
  * V step:  G_U = sum_k U_k^T U_k (r x r) and W^^T U = sum_k W^_k^T U_k (n x r); then
             V = (W^^T U + rho (Z_V - L_V)) G_U^-1 and SVID(V) are replicated
  * objective: ||W^||^2 - 2 <W^^T U, V> + <U^T U, V^T V> from the replicated sums
  * finish:  ||U_:k||^2 = sum_k ||U_k,:k||^2 (r values) for the balancing gains, and the
             reconstruction error's sum of squares (one scalar).
Each rank here runs that decomposition in FP64 with torch.distributed all-reduces (gloo,
two ranks, 127.0.0.1); the gathered result must equal the unsharded FP64 oracle's
(oracle.lbadmm) to rounding: scales 1e-9 relative, packed signs bit for bit, the
per-iteration objective and the final error 1e-10 relative.  On GPUs the same sums are
NCCL all-reduces over NVLink of device buffers between the library's kernels, no TMA
multicast anywhere.
"""
import os
import socket
import sys

import numpy as np
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
M, N, R, ITERS, K, RHO, LAM = 48, 40, 6, 12, 4, 1.0, 1e-4


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _weight():
    rng = np.random.default_rng(7)
    d_out = np.exp(0.3 * rng.standard_normal(M))
    d_in = np.exp(0.3 * rng.standard_normal(N))
    return rng.standard_normal((M, N)), d_in, d_out


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime

    import torch
    import torch.distributed as dist

    from oracle import lbadmm as O

    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))

    def allsum(x):
        t = torch.as_tensor(np.asarray(x, dtype=np.float64)).clone()
        dist.all_reduce(t)
        return t.numpy()

    W, d_in, d_out = _weight()
    rows = np.array_split(np.arange(M), world)[rank]
    Wt_k = d_out[rows, None] * W[rows] * d_in[None, :]                  # W~_k
    gamma = np.sqrt(allsum(np.sum(Wt_k * Wt_k))) / (2.0 * np.sqrt(R))
    Wh_k = Wt_k / gamma
    w2 = allsum(np.sum(Wh_k * Wh_k))
    V = O.init_latent(N, R, 0)                                          # replicated
    mk = len(rows)
    U_k = np.zeros((mk, R))
    ZU, LU = np.zeros((mk, R)), np.zeros((mk, R))
    ZV, LV = np.zeros((N, R)), np.zeros((N, R))
    c = LAM + RHO
    objective = []
    for _ in range(ITERS):
        # U step: local rows, replicated V
        GV = V.T @ V + c * np.eye(R)
        U_k = np.linalg.solve(GV, (Wh_k @ V + RHO * (ZU - LU)).T).T
        # SVID(U): power steps with the column sums and the norm all-reduced
        A = np.abs(U_k + LU)
        b = np.ones(R)
        a = np.zeros(mk)
        for _ in range(K):
            t = A @ b
            nt = float(np.sqrt(allsum(np.sum(t * t))))
            if nt == 0.0:
                a, b = np.zeros(mk), np.zeros(R)
                break
            a = t / nt
            b = allsum(A.T @ a)
        ZU = O.sign_pm(U_k + LU) * np.outer(a, b)
        LU = LU + U_k - ZU
        # V step: Gram of U and W^^T U summed over ranks, the rest replicated
        GU = allsum(U_k.T @ U_k) + c * np.eye(R)
        P = allsum(Wh_k.T @ U_k)
        V = np.linalg.solve(GU, (P + RHO * (ZV - LV)).T).T
        ZV, _, _ = O.svid(V + LV, K)
        LV = LV + V - ZV
        objective.append(float((w2 - 2.0 * np.sum(P * V) + np.sum((GU - c * np.eye(R)) * (V.T @ V)))
                               / w2))
    # finish: balancing gains from the summed column norms, local scales and signs
    nu = np.sqrt(allsum(np.sum(U_k * U_k, axis=0)))
    nv = np.linalg.norm(V, axis=0)
    g = np.ones(R)
    ok = (nu > 0) & (nv > 0)
    g[ok] = np.sqrt(nv[ok] / nu[ok])
    Ub, Vb = U_k * g[None, :], V / g[None, :]
    s1_k = gamma * np.abs(Ub).mean(axis=1)
    s2 = np.abs(Vb).mean(axis=1)
    D = Wt_k - (s1_k[:, None] * (O.sign_pm(Ub) @ O.sign_pm(Vb).T)) * s2[None, :]
    rel_err = float(np.sqrt(allsum(np.sum(D * D)) / allsum(np.sum(Wt_k * Wt_k))))
    np.savez(os.path.join(out_dir, f"rank{rank}.npz"), rows=rows, s1=s1_k, s2=s2,
             Up=O.pack_signs(Ub), Vp=O.pack_signs(Vb), objective=np.array(objective),
             rel_err=rel_err)
    dist.barrier()
    dist.destroy_process_group()


def test_row_sharded_iteration_equals_the_unsharded_oracle(tmp_path):
    sys.path.insert(0, ROOT)
    from oracle import lbadmm as O
    world, port = 2, _free_port()
    mp.start_processes(_rank_main, args=(world, port, str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    parts = [np.load(tmp_path / f"rank{k}.npz") for k in range(world)]
    W, d_in, d_out = _weight()
    ref = O.lbadmm(W, d_in, d_out, r=R, rho=RHO, lam=LAM, iters=ITERS, K=K, seed=0)
    s1 = np.concatenate([p["s1"] for p in parts])
    Up = np.concatenate([p["Up"] for p in parts])
    assert np.max(np.abs(s1 - ref.s1)) <= 1e-9 * np.max(np.abs(ref.s1))
    for p in parts:
        assert np.max(np.abs(p["s2"] - ref.s2)) <= 1e-9 * np.max(np.abs(ref.s2))
        np.testing.assert_array_equal(p["Vp"], ref.V_packed)
        np.testing.assert_allclose(p["objective"], ref.objective, rtol=1e-10)
        assert abs(float(p["rel_err"]) - ref.rel_err) <= 1e-10 * ref.rel_err
    np.testing.assert_array_equal(Up, ref.U_packed)
