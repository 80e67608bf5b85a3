"""GPU parity of the calibration preconditioners against the FP64 oracle."""
import numpy as np
import pytest
import torch

from conftest import max_rel
from oracle import calib as O
from synth import CALIB_TOKENS, planted_problem, stream_chunks, stream_tensor

pytestmark = pytest.mark.gpu
TOL_D = 1e-5      # preconditioner diagonals, relative per element


def _rel(x, ref):
    x = np.asarray(x, dtype=np.float64)
    return float(np.max(np.abs(x - ref) / np.abs(ref)))


def test_planted_config_fp32_streams(nq):
    p = planted_problem(0)
    d_in, d_out, a_in, a_out = nq.nq_calib_precond(p["acts"].cuda(), p["grads"].cuda())
    r_in, r_out, ra_in, ra_out = O.calib_precond([p["acts"].numpy()], [p["grads"].numpy()])
    assert _rel(d_in.cpu(), r_in) < TOL_D
    assert _rel(d_out.cpu(), r_out) < TOL_D
    assert abs(a_in - ra_in) <= 1e-6 * ra_in + 1e-12
    assert abs(a_out - ra_out) <= 1e-6 * ra_out + 1e-12


@pytest.mark.parametrize("T,C,dtype", [(5000, 1000, torch.bfloat16), (4097, 1001, torch.bfloat16),
                                       (300, 257, torch.float32), (1, 8, torch.bfloat16),
                                       (1, 1, torch.float32), (70000, 24, torch.bfloat16),
                                       (333, 4096, torch.float32)])
def test_moments_ragged_shapes(nq, T, C, dtype):
    x = torch.cat(list(stream_chunks(T * 7 + C, "x", T, C, dtype=dtype)))
    s, q = nq.nq_calib_stats(x.cuda())
    rs, rq, _ = O.channel_moments([x.float().numpy()])
    assert _rel(s.cpu(), rs) < 1e-6
    assert _rel(q.cpu(), rq) < 1e-6


def test_zero_channel_constant_channels_and_override(nq):
    T = 4096
    x = torch.randn(T, 64)
    x[:, 3] = 0.0
    x[:, 5] = torch.where(torch.rand(T) < 0.5, -2.0, 2.0)
    g = torch.randn(T, 32) * 3
    d_in, d_out, a_in, _ = nq.nq_calib_precond(x.cuda(), g.cuda())
    r_in, r_out, ra, _ = O.calib_precond([x.numpy()], [g.numpy()])
    assert _rel(d_in.cpu(), r_in) < TOL_D and _rel(d_out.cpu(), r_out) < TOL_D
    d_fix, _, a_fix, _ = nq.nq_calib_precond(x.cuda(), g.cuda(), alpha_override=0.25)
    r_fix, _, _, _ = O.calib_precond([x.numpy()], [g.numpy()], alpha_override=0.25)
    assert a_fix == 0.25 and _rel(d_fix.cpu(), r_fix) < TOL_D
    # constant |x| per channel: Ledoit-Wolf intensity 0, d = |x|
    c = torch.where(torch.rand(T, 16) < 0.5, -1.0, 1.0) * torch.arange(1, 17).float()
    dc, _, ac, _ = nq.nq_calib_precond(c.cuda(), c.cuda())
    assert ac == 0.0
    np.testing.assert_allclose(dc.cpu().numpy(), np.arange(1, 17), rtol=1e-6)


def test_nonfinite_stream_is_reported(nq):
    x = torch.randn(100, 16)
    x[7, 3] = float("nan")
    with pytest.raises(nq.NQError) as e:
        nq.nq_calib_precond(x.cuda(), torch.randn(100, 8).cuda())
    assert e.value.code == 4


def test_full_size_bf16_streams_are_deterministic_and_match(nq):
    # 128 x 2048 calibration tokens over a 4096-channel layer input (the Llama-2-7B q_proj
    # workload); the oracle streams the same seeded chunks in FP64.
    T, C = CALIB_TOKENS, 4096
    acts = stream_tensor(0, "acts", T, C).cuda()
    grads = stream_tensor(0, "grads", T, C).cuda()
    d_in, d_out, a_in, a_out = nq.nq_calib_precond(acts, grads)
    d_in2, d_out2, _, _ = nq.nq_calib_precond(acts, grads)
    assert torch.equal(d_in, d_in2) and torch.equal(d_out, d_out2)
    del acts, grads
    r_in, r_out, ra_in, ra_out = O.calib_precond(
        (c.float().numpy() for c in stream_chunks(0, "acts", T, C)),
        (c.float().numpy() for c in stream_chunks(0, "grads", T, C)))
    assert _rel(d_in.cpu(), r_in) < TOL_D
    assert _rel(d_out.cpu(), r_out) < TOL_D
    assert abs(a_in - ra_in) <= 1e-5 * ra_in
