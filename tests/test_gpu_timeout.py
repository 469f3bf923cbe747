"""The bounded device-side wait gives up and reports BCJR_ERR_TIMEOUT, and the
GPU keeps answering (needs a B200).

The cluster teams' exchange waits on mbarriers with a bounded wait.  The
option `timeout_probe_cycles` makes a call run that same wait, before any
exchange between the cluster's CTAs starts, on an mbarrier that nothing
arrives at, bounded at a few hundred cycles: the wait must give up, the status
word must read BCJR_ERR_TIMEOUT, and the next normal call on the same device
must still match the oracle.  Nothing faults or hangs: the wait is bounded and
no transfer is in flight when the kernel returns.
"""
import numpy as np
import pytest
import torch

import bcjr_inputs as I
import oracle
from parity import LOGZ_ATOL_PER_STEP, LOGZ_RTOL, W_HAT_ATOL, assert_abs, to_np

pytestmark = pytest.mark.gpu

TIMEOUT = 5


@pytest.mark.parametrize("L", [14, 16])
def test_bounded_wait_gives_up_and_the_device_still_answers(L):
    import differentiable_bcjr_b200 as B
    dev = torch.device("cuda", 0)
    k, n, N, T = 2, 8, 2, 0.3
    c, w = I.codebook(1 << L, seed=70 + L), I.weights(N, n, seed=80 + L)
    dc, dw = c.to(dev), w.to(dev)
    ws = B.Workspace(dev)
    B.bcjr_forward(dw, dc, T, L, k, ws=ws, timeout_probe_cycles=300)
    assert B.get_status(ws.buf) == TIMEOUT
    w_hat, _, log_z = B.bcjr_forward(dw, dc, T, L, k, ws=ws)
    assert B.get_status(ws.buf) == 0
    o_what, o_lz, _ = oracle.forward(w, c, T, L, k)
    assert_abs(w_hat, o_what, W_HAT_ATOL, "w_hat after a timed-out call")
    np.testing.assert_allclose(to_np(log_z), o_lz, rtol=LOGZ_RTOL, atol=LOGZ_ATOL_PER_STEP * n)


def test_negative_probe_bound_is_rejected():
    import differentiable_bcjr_b200 as B
    dev = torch.device("cuda", 0)
    w, c = I.weights(2, 4, seed=1).to(dev), I.codebook(1 << 8, seed=2).to(dev)
    with pytest.raises(B.BCJRError) as err:
        B.bcjr_forward(w, c, 0.5, 8, 2, timeout_probe_cycles=-1)
    assert err.value.status == 1
