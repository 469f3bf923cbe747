"""bcjr_forward_static_scratch (the entry point whose scratch is a static device
array, so that it allocates nothing) against bcjr_forward with a workspace and
against the float64 oracle, with its device-side status read through
bcjr_static_scratch_status.

The file name sorts last so that the test also runs after every other GPU test
in the same process; it passes alone as well."""
import numpy as np
import pytest
import torch

import bcjr_inputs as I
import oracle
from parity import LOGZ_ATOL_PER_STEP, LOGZ_RTOL, MARGINAL_ATOL, W_HAT_ATOL, assert_abs, to_np

pytestmark = pytest.mark.gpu

# (state_bits, k, seq_len, n_seq, T): small problems whose forward workspace
# fits in the static scratch; the second shape reuses the scratch at another size.
SHAPES = [(10, 2, 64, 8, 0.3), (12, 3, 40, 3, 0.1), (8, 2, 256, 100, 0.05)]


def _inputs(L, k, n, N, dev):
    c = I.codebook(1 << L, seed=4000 + L).to(dev)
    w = I.weights(N, n, seed=5000 + L).to(dev)
    return w, c


@pytest.mark.parametrize("L,k,n,N,T", SHAPES)
def test_static_scratch_matches_workspace_path(L, k, n, N, T):
    import differentiable_bcjr_b200 as B
    dev = torch.device("cuda", 0)
    w, c = _inputs(L, k, n, N, dev)
    need = B.workspace_size(B.OP_FORWARD, L, k, n, N)
    assert 0 < need <= B.STATIC_SCRATCH_BYTES
    ref_what, ref_marg, ref_lz = B.bcjr_forward(w, c, T, L, k, want_marginals=True)
    o_what, o_lz, o_gamma = oracle.forward(w.cpu(), c.cpu(), T, L, k, want_gamma=True)
    for _ in range(2):  # two calls in a row on the same scratch
        w_hat = torch.full_like(ref_what, float("nan"))
        log_z = torch.full_like(ref_lz, float("nan"))
        marg = torch.full_like(ref_marg, float("nan"))
        B.bcjr_forward_static_scratch(w, c, T, L, k, w_hat, log_z=log_z, marginals=marg)
        assert B.static_scratch_status(dev) == 0
        assert_abs(w_hat, to_np(ref_what), W_HAT_ATOL, "w_hat")
        assert_abs(marg, to_np(ref_marg), MARGINAL_ATOL, "marginals")
        torch.testing.assert_close(log_z, ref_lz, rtol=LOGZ_RTOL, atol=0.0)
        assert_abs(w_hat, o_what, W_HAT_ATOL, "w_hat vs oracle")
        assert_abs(marg, o_gamma, MARGINAL_ATOL, "marginals vs oracle")
        np.testing.assert_allclose(to_np(log_z), o_lz, rtol=LOGZ_RTOL, atol=LOGZ_ATOL_PER_STEP * n)


def test_static_scratch_status_reports_a_nonfinite_input():
    import differentiable_bcjr_b200 as B
    dev = torch.device("cuda", 0)
    L, k, n, N, T = 10, 2, 16, 3, 0.3
    w, c = _inputs(L, k, n, N, dev)
    w[1, 5] = float("inf")
    w_hat = torch.empty((N, n), device=dev)
    log_z = torch.empty((N,), device=dev)
    B.bcjr_forward_static_scratch(w, c, T, L, k, w_hat, log_z=log_z)
    assert B.static_scratch_status(dev) == 6  # BCJR_ERR_NONFINITE, from the device-side word
    w[1, 5] = 0.25
    B.bcjr_forward_static_scratch(w, c, T, L, k, w_hat, log_z=log_z)
    assert B.static_scratch_status(dev) == 0  # cleared by the next call


def test_static_scratch_checks_output_shapes():
    import differentiable_bcjr_b200 as B
    dev = torch.device("cuda", 0)
    L, k, n, N, T = 8, 2, 16, 4, 0.3
    w, c = _inputs(L, k, n, N, dev)
    w_hat = torch.empty((N, n), device=dev)
    with pytest.raises(ValueError):
        B.bcjr_forward_static_scratch(w, c, T, L, k, w_hat, marginals=torch.empty((N, n), device=dev))
    with pytest.raises(ValueError):
        B.bcjr_forward_static_scratch(w, c[:100].contiguous(), T, L, k, w_hat)
    with pytest.raises(ValueError):
        B.bcjr_forward_static_scratch(w, c, T, L, k, torch.empty((N, n), device=dev, dtype=torch.float64))
    with pytest.raises(ValueError):
        B.bcjr_forward_static_scratch(w, c, T, L, k, w_hat, log_z=torch.empty((N + 1,), device=dev))


def test_static_scratch_rejects_oversized_problem():
    import differentiable_bcjr_b200 as B
    dev = torch.device("cuda", 0)
    L, k, n, N = 16, 2, 256, 4
    assert B.workspace_size(B.OP_FORWARD, L, k, n, N) > B.STATIC_SCRATCH_BYTES
    w, c = _inputs(L, k, n, N, dev)
    w_hat = torch.full((N, n), 7.0, device=dev)
    with pytest.raises(B.BCJRError) as err:
        B.bcjr_forward_static_scratch(w, c, 0.3, L, k, w_hat)
    assert err.value.status == 3  # BCJR_ERR_WORKSPACE, found before any launch
    torch.cuda.synchronize()
    assert bool((w_hat == 7.0).all())  # nothing was written


def test_static_scratch_allocates_nothing():
    import differentiable_bcjr_b200 as B
    dev = torch.device("cuda", 0)
    L, k, n, N, T = 10, 2, 64, 8, 0.3
    w, c = _inputs(L, k, n, N, dev)
    w_hat = torch.empty((N, n), device=dev)
    log_z = torch.empty((N,), device=dev)
    B.bcjr_forward_static_scratch(w, c, T, L, k, w_hat, log_z=log_z)  # first call: per-device set-up
    torch.cuda.synchronize()
    free_before, _ = torch.cuda.mem_get_info(dev)
    for _ in range(3):
        B.bcjr_forward_static_scratch(w, c, T, L, k, w_hat, log_z=log_z)
    torch.cuda.synchronize()
    free_after, _ = torch.cuda.mem_get_info(dev)
    assert free_after == free_before
