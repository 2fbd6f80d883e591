"""Failure detection on the GPU without a fault: a wait that runs out ends
its launch with CCE_STATUS_TIMEOUT (no trap, no hang), the stream and the
context stay usable, and the opt-in status check turns device-reported
errors into exceptions."""
import numpy as np
import pytest
import torch

import oracle
from linear_cross_entropy_cce_b200 import cce, synthetic as syn
from linear_cross_entropy_cce_b200.autograd import linear_cross_entropy
from _helpers import TOL_GRAD, TOL_ROW, normwise, to_np, upload

pytestmark = pytest.mark.gpu


def test_wait_that_never_completes_times_out_and_the_stream_stays_usable():
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    cce.debug_stall(1_000_000, st)  # the stage it waits for is never filled: 1 ms limit
    torch.cuda.synchronize()
    assert int(st.item()) == cce.STATUS_TIMEOUT
    with pytest.raises(cce.CCEError, match="TIMEOUT"):
        cce.check_status(st)
    # the next calls on the same stream compute correctly
    x = syn.make_inputs(syn.WORKLOADS["tiny"], seed=5)
    H, segs, y = upload(x)
    st2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    loss, lse = cce.fwd(H, segs[0][2], y, x.ignore_index, status=st2)
    torch.cuda.synchronize()
    assert cce.check_status(st2) == 0
    rl, rs = oracle.forward(x.H, x.segments, x.y, x.wl.V, x.ignore_index)
    assert np.max(np.abs(to_np(loss) - rl)) <= TOL_ROW
    assert np.max(np.abs(to_np(lse) - rs)) <= TOL_ROW


def test_wait_on_a_cta_pair_times_out_and_the_stream_stays_usable():
    """The CTA-pair kernels' abort path: both CTAs give up, free the pair's
    tensor memory and return; the following pair-kernel calls are correct."""
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    cce.debug_stall(1_000_000, st, pair=True)
    torch.cuda.synchronize()
    assert int(st.item()) == cce.STATUS_TIMEOUT
    # an unfiltered forward + backward: every tensor-core kernel on CTA pairs
    x = syn.make_inputs(syn.WORKLOADS["tiny"], seed=7)
    H, segs, y = upload(x)
    st2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    loss, lse = cce.fwd(H, segs[0][2], y, x.ignore_index, status=st2)
    dl = torch.from_numpy(x.dloss_mean()).cuda()
    dH, dE, _ = cce.bwd(H, segs[0][2], y, lse, dl, x.ignore_index, status=st2)
    torch.cuda.synchronize()
    assert cce.check_status(st2) == 0
    rl, rs = oracle.forward(x.H, x.segments, x.y, x.wl.V, x.ignore_index)
    assert np.max(np.abs(to_np(loss) - rl)) <= TOL_ROW
    rH, rE = oracle.backward(x.H, x.segments, x.y, x.wl.V, x.dloss_mean(), x.ignore_index)[:2]
    assert normwise(to_np(dH), rH) <= TOL_GRAD
    assert normwise(to_np(dE), rE[0] if isinstance(rE, (list, tuple)) else rE) <= TOL_GRAD


def test_stall_argument_checks():
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    L = cce.lib()
    assert L.cce_debug_stall(0, st.data_ptr(), None) == cce.CCE_EINVAL
    assert L.cce_debug_stall(2_000_000_000, st.data_ptr(), None) == cce.CCE_EINVAL
    assert L.cce_debug_stall(1000, None, None) == cce.CCE_EINVAL
    assert L.cce_debug_stall_pair(0, st.data_ptr(), None) == cce.CCE_EINVAL
    assert L.cce_debug_stall_pair(1000, None, None) == cce.CCE_EINVAL


def test_status_check_raises_on_a_bad_target():
    x = syn.make_inputs(syn.WORKLOADS["tiny"], seed=6)
    x.y[4] = x.wl.V + 3
    H, segs, y = upload(x)
    Hl = H.detach().clone().requires_grad_(True)
    E = segs[0][2].detach().clone().requires_grad_(True)
    with pytest.raises(cce.CCEError, match="BADTARGET"):
        linear_cross_entropy(Hl, E, y, check_status=True)
    # without the check the row is NaN and nothing raises
    loss = linear_cross_entropy(Hl, E, y, reduction="none")
    assert torch.isnan(loss[4]) and not torch.isnan(loss[:4]).any()
