"""GPU parity of the binary GEMV/GEMM on the packed factors against the FP64 oracle.

Sign decoding is checked bit-exactly (identity inputs return the reconstructed layer,
whose signs the oracle fixes); values within 1e-5 of the oracle relative to the largest
output, for the packed-bit path (B <= 16) and the tensor-core path (B > 16), on FP32
and BF16 inputs, ragged sizes and ranks that are not multiples of 32.
"""
import numpy as np
import pytest
import torch

from conftest import max_rel
from oracle import binary as OB
from oracle import lbadmm as O
from oracle.splitmix import sign_matrix

pytestmark = pytest.mark.gpu
TOL = 1e-5


def _layer(m, n, r, seed):
    rng = np.random.default_rng(seed)
    Us = sign_matrix(seed, m, r)
    Vs = sign_matrix(seed + 7, n, r)
    s1 = np.exp(0.5 * rng.standard_normal(m)).astype(np.float32)
    s2 = (np.exp(0.5 * rng.standard_normal(n)) / np.sqrt(r)).astype(np.float32)
    Up, Vp = O.pack_signs(Us), O.pack_signs(Vs)
    dev = [torch.from_numpy(a.view(np.int32)).cuda() for a in (Up, Vp)]
    return Up, Vp, s1, s2, dev[0], dev[1], torch.from_numpy(s1).cuda(), torch.from_numpy(s2).cuda()


@pytest.mark.parametrize("B", [1, 3, 16, 64, 200])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("m,n,r", [(300, 257, 33), (1000, 777, 130), (129, 512, 1)])
def test_binary_matmul_matches_oracle(nq, B, dtype, m, n, r):
    Up, Vp, s1, s2, Upd, Vpd, s1d, s2d = _layer(m, n, r, m + n + r + B)
    X = torch.randn(B, n, generator=torch.Generator().manual_seed(B)).to(dtype)
    Y = nq.nq_binary_matmul(Upd, Vpd, s1d, s2d, r, X.cuda()).cpu().double().numpy()
    ref = OB.binary_matmul(X.double().numpy(), Up, Vp, s1, s2, r)
    assert max_rel(Y, ref) <= TOL


@pytest.mark.parametrize("path_B", [1, 32])
def test_identity_inputs_decode_the_signs_exactly(nq, path_B):
    # with X = I (and s1 = s2 = 1) row j of Y is row j of V+- U+-^T: small integers,
    # computed exactly by both paths
    m, n, r = 70, 40, 45
    Up, Vp, _, _, Upd, Vpd, _, _ = _layer(m, n, r, 11)
    ones_m, ones_n = torch.ones(m, device="cuda"), torch.ones(n, device="cuda")
    Y = torch.cat([nq.nq_binary_matmul(Upd, Vpd, ones_m, ones_n, r,
                                       torch.eye(n, device="cuda")[j:j + path_B])
                   for j in range(0, n, path_B)]).cpu().numpy()
    ref = O.unpack_signs(Vp, r) @ O.unpack_signs(Up, r).T
    np.testing.assert_array_equal(Y[:n], ref)


def test_layer_from_lbadmm_applies_like_its_reconstruction(nq):
    # end to end: factorise a layer, then apply the packed result to a batch of inputs
    m, n, r = 512, 384, 96
    W = torch.randn(m, n) * 0.02
    res = nq.nq_lbadmm(W.cuda(), r, iters=10)
    X = torch.randn(40, n)
    for B in (1, 40):
        Y = nq.nq_binary_matmul(res["U_packed"], res["V_packed"], res["s1"], res["s2"], r,
                                X[:B].cuda()).cpu().double().numpy()
        Up = res["U_packed"].cpu().numpy().view(np.uint32)
        Vp = res["V_packed"].cpu().numpy().view(np.uint32)
        Wq = O.reconstruct(res["s1"].cpu().double().numpy(), O.unpack_signs(Up, r),
                           O.unpack_signs(Vp, r), res["s2"].cpu().double().numpy())
        assert max_rel(Y, X[:B].double().numpy() @ Wq.T) <= TOL
