"""Warm start of V from a similar layer (summary page, weaknesses section: a warm-start
strategy that carries the initialisation over from similar layers).

The step-level interface takes it as it stands: prepare the new layer, write the other
layer's latent V into the state, re-derive the operand copies, iterate.  The oracle's
LB-ADMM takes the same V_0 (``oracle.lbadmm.lbadmm(..., V0=...)``).  Checked: the GPU run
from the warm start matches the oracle's from the same V_0 within 1 % (final reconstruction
error and every iteration's objective), and the warm start is ahead of the seeded start
after the same number of iterations.
"""
import numpy as np
import pytest
import torch

from oracle import lbadmm as O
from synth import student_t_weight

pytestmark = pytest.mark.gpu


def test_warm_start_from_a_similar_layer(nq):
    m, n, r = 1024, 768, 128
    W1 = student_t_weight(11, "layer_a", m, n).float()
    g = torch.Generator().manual_seed(12)
    W2 = (W1 + 0.2 * W1.std() * torch.randn(m, n, generator=g)).to(torch.bfloat16)
    st1 = nq.LBState(m, n, r)
    st1.prepare(W1.to(torch.bfloat16).cuda())
    st1.iterate(30, want_objective=False)
    V1 = st1.field("V")[:, :r].float().clone()

    iters = 10
    warm = nq.LBState(m, n, r)
    warm.prepare(W2.cuda())
    warm.field("V")[:, :r].copy_(V1)
    warm.sync_operands()
    obj_w = np.array(warm.iterate(iters))
    err_w = warm.finish(W2.cuda())["rel_err"]
    assert warm.check_device_error() == 0

    ref = O.lbadmm(W2.double().numpy(), r=r, iters=iters, V0=V1.cpu().double().numpy())
    assert abs(err_w - ref.rel_err) <= 0.01 * ref.rel_err
    np.testing.assert_allclose(obj_w, ref.objective, rtol=0.01)

    cold = nq.LBState(m, n, r)
    cold.prepare(W2.cuda())
    obj_c = np.array(cold.iterate(iters))
    assert obj_w[-1] < obj_c[-1]
