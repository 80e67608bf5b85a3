"""Device-side error paths end with a status the host reads, and the context stays usable.

The library's waits are bounded and its numerical checks raise a status instead of
trapping.  nq_selftest runs two of these paths on purpose: the bounded counter wait of
the Cholesky dataflow on a word that nothing sets (it must give up and report
NQ_ERR_TIMEOUT), and the cooperative Cholesky kernel on G = -I (it must report
NQ_ERR_NOT_SPD).  After each, ordinary library calls on the same context must succeed
and agree with the oracle.
"""
import numpy as np
import pytest
import torch

from oracle import lbadmm as O
from rank_binary_factorization_b200 import _lib

pytestmark = pytest.mark.gpu


def _context_usable(nq):
    rng = np.random.default_rng(3)
    X = rng.standard_normal((77, 45)).astype(np.float32)
    bits = nq.nq_pack_signs(torch.from_numpy(X).cuda())
    torch.cuda.synchronize()
    np.testing.assert_array_equal(bits.cpu().numpy().view(np.uint32), O.pack_signs(X))
    res = nq.nq_lbadmm(torch.randn(96, 64).cuda(), 8, iters=3)
    assert np.isfinite(res["rel_err"]) and 0.0 < res["rel_err"] < 1.0


def test_wait_timeout_is_reported(nq):
    assert nq.nq_selftest("wait_timeout") == _lib.NQ_ERR_TIMEOUT
    _context_usable(nq)


def test_not_spd_is_reported(nq):
    assert nq.nq_selftest("not_spd") == _lib.NQ_ERR_NOT_SPD
    _context_usable(nq)


def test_selftest_arguments(nq):
    ws = nq.workspace(nq.lib.nq_selftest_workspace_size())
    stream = torch.cuda.current_stream().cuda_stream
    import ctypes
    assert nq.lib.nq_selftest(7, ctypes.c_void_p(ws.data_ptr()), ws.numel(),
                              ctypes.c_void_p(stream)) == _lib.NQ_ERR_INVALID_ARG
    assert nq.lib.nq_selftest(0, ctypes.c_void_p(ws.data_ptr()), 16,
                              ctypes.c_void_p(stream)) == _lib.NQ_ERR_WORKSPACE
