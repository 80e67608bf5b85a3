"""The allocation-free calibration entry point (nq_calib_stats_noalloc).

Callers that cannot allocate device memory or pass a workspace (for example a plugin
inside a host program that owns the device memory pool) use this variant, whose scratch
is a fixed array inside the library.  Checked here through the C ABI on two calls in a
row (so that anything the first call leaves in the shared array cannot leak into the
second): bit for bit against the workspace-based nq_calib_stats, which runs the same
reduction in the same order, and against the FP64 oracle's channel moments at 1e-6.
This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

from oracle import calib as OC

pytestmark = pytest.mark.gpu


def _noalloc(nq, X):
    T, C = X.shape
    s = torch.empty(C, dtype=torch.float64, device=X.device)
    q = torch.empty(C, dtype=torch.float64, device=X.device)
    dt = nq.NQ_BF16 if X.dtype == torch.bfloat16 else nq.NQ_F32
    code = nq.lib.nq_calib_stats_noalloc(ctypes.c_void_p(X.data_ptr()), T, C, dt,
                                         ctypes.c_void_p(s.data_ptr()),
                                         ctypes.c_void_p(q.data_ptr()),
                                         ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return code, s, q


def test_noalloc_matches_workspace_entry_on_two_calls_in_a_row(nq):
    g = torch.Generator().manual_seed(11)
    cases = [torch.randn(70000, 4096, generator=g).to(torch.bfloat16),
             (torch.randn(3000, 1000, generator=g) * 3).to(torch.float32)]
    for X in cases:
        s_o, q_o, _ = OC.channel_moments([X.float().numpy()])
        X = X.cuda()
        code, s, q = _noalloc(nq, X)
        assert code == 0, nq.status_string(code)
        s_ref, q_ref = nq.nq_calib_stats(X)
        torch.cuda.synchronize()
        assert torch.equal(s, s_ref) and torch.equal(q, q_ref)
        for a, b in ((s, s_o), (q, q_o)):
            a = a.cpu().numpy()
            assert np.max(np.abs(a - b) / np.abs(b)) < 1e-6


def test_noalloc_rejects_sizes_beyond_its_scratch(nq):
    X = torch.zeros(2, 40000, dtype=torch.bfloat16, device="cuda")
    code, _, _ = _noalloc(nq, X)
    assert code == 7     # NQ_ERR_UNSUPPORTED: more channels than the fixed scratch serves
