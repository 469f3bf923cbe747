"""GPU parity with the float64 oracle through the C ABI (needs a B200).

Shapes cover every kernel instantiation: k = 1..4, teams narrower than a
warp (state_bits <= 8), single-CTA teams (state_bits 9..13, up to 512
threads), and thread-block clusters of 2, 4 and 8 CTAs of 512 threads
(state_bits = 14, 15, 16); ragged sequence lengths; checkpoint intervals
C > 1 that do and do not divide the length; the degenerate n = 1 and N = 0;
marginals of every team shape, clusters included.
"""
import numpy as np
import pytest
import torch

import bcjr_inputs as I
import oracle
from parity import (GRAD_REL_L2, LOGZ_RTOL, MARGINAL_ATOL, W_HAT_ATOL, assert_abs, assert_rel_l2,
                    to_np)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    import differentiable_bcjr_b200 as B
    B.lib()
    return B


def _case(L, k, n, N, seed):
    S = 1 << L
    return (I.codebook(S, seed=1000 + seed), I.weights(N, n, seed=2000 + seed),
            I.upstream_grad(N, n, seed=3000 + seed))


def _run_fwd_bwd(B, L, k, n, N, T, seed, C=0, marginals=False):
    c, w, g = _case(L, k, n, N, seed)
    dc, dw, dg = c.cuda(), w.cuda(), g.cuda()
    w_hat, marg, log_z = B.bcjr_forward(dw, dc, T, L, k, want_marginals=marginals, checkpoint_interval=C)
    grad_w, grad_c = B.bcjr_backward(dg, dw, dc, w_hat, T, L, k, checkpoint_interval=C)
    torch.cuda.synchronize()
    return (c, w, g), (w_hat, marg, log_z, grad_w, grad_c)


SHAPES = [
    # L, k, n, N, T
    (4, 1, 9, 3, 0.7),
    (4, 2, 5, 5, 0.4),
    (6, 3, 7, 3, 0.9),
    (8, 4, 6, 2, 0.6),
    (8, 2, 64, 16, 0.5),      # the tiny workload: L=8, k=2, n=64, 16 sequences
    (9, 2, 11, 3, 0.3),       # 32-thread teams
    (10, 1, 13, 2, 1.1),
    (11, 3, 9, 3, 0.25),
    (12, 4, 8, 2, 0.8),
    (13, 2, 10, 2, 0.15),     # 512-thread CTA
    (14, 3, 7, 2, 0.5),       # 2-CTA cluster
    (15, 2, 6, 2, 0.35),      # 4-CTA cluster
    (16, 2, 5, 2, 0.2),       # 8-CTA cluster
    (16, 3, 4, 2, 0.1),
    (16, 4, 4, 2, 0.1),
]


@pytest.mark.parametrize("L,k,n,N,T", SHAPES)
def test_forward_backward_parity(B, L, k, n, N, T):
    (c, w, g), (w_hat, marg, log_z, grad_w, grad_c) = _run_fwd_bwd(B, L, k, n, N, T, seed=L * 7 + k,
                                                                  marginals=(L <= 12))
    o_what, o_lz, o_gamma = oracle.forward(w, c, T, L, k, want_gamma=(L <= 12))
    o_gw, o_gc = oracle.backward(g, w, c, T, L, k)
    assert_abs(w_hat, o_what, W_HAT_ATOL, "w_hat")
    np.testing.assert_allclose(to_np(log_z), o_lz, rtol=LOGZ_RTOL, atol=1e-4)
    if marg is not None:
        assert_abs(marg, o_gamma, MARGINAL_ATOL, "marginals")
    assert_rel_l2(grad_w, o_gw, GRAD_REL_L2, "grad_w")
    assert_rel_l2(grad_c, o_gc, GRAD_REL_L2, "grad_codebook")


@pytest.mark.parametrize("L,k,n,N,T", [(14, 2, 9, 2, 0.3), (15, 2, 12, 2, 0.2), (16, 2, 10, 2, 0.1),
                                         (16, 2, 8, 3, 0.01), (16, 1, 6, 2, 0.4), (16, 3, 6, 2, 0.3),
                                         (16, 4, 5, 2, 0.5), (15, 4, 7, 2, 0.25)])
def test_cluster_team_marginals(B, L, k, n, N, T):
    # the marginal-store instantiation of the 2-, 4- and 8-CTA cluster kernels
    c, w, _ = _case(L, k, n, N, seed=600 + L * 5 + k)
    w_hat, marg, log_z = B.bcjr_forward(w.cuda(), c.cuda(), T, L, k, want_marginals=True)
    o_what, o_lz, o_gamma = oracle.forward(w, c, T, L, k, want_gamma=True)
    assert_abs(marg, o_gamma, MARGINAL_ATOL, f"marginals L={L} k={k}")
    assert_abs(w_hat, o_what, W_HAT_ATOL, f"w_hat L={L} k={k}")
    np.testing.assert_allclose(to_np(log_z), o_lz, rtol=LOGZ_RTOL, atol=1e-4)


@pytest.mark.parametrize("L,k,nseq", [(16, 2, 2), (16, 2, 3), (16, 2, 4), (15, 3, 3), (14, 4, 4)])
def test_sequences_in_flight(B, L, k, nseq):
    # the forward call with 2, 3 or 4 sequences in flight per cluster team, on a
    # batch that leaves the last round of teams partly idle
    n, N, T = 9, 7, 0.2
    c, w, _ = _case(L, k, n, N, seed=700 + nseq)
    w_hat, marg, log_z = B.bcjr_forward(w.cuda(), c.cuda(), T, L, k, want_marginals=True,
                                        sequences_in_flight=nseq)
    o_what, o_lz, o_gamma = oracle.forward(w, c, T, L, k, want_gamma=True)
    assert_abs(w_hat, o_what, W_HAT_ATOL, f"w_hat nseq={nseq}")
    assert_abs(marg, o_gamma, MARGINAL_ATOL, f"marginals nseq={nseq}")
    np.testing.assert_allclose(to_np(log_z), o_lz, rtol=LOGZ_RTOL, atol=1e-4)


@pytest.mark.parametrize("L,k,n,N,T,C", [(8, 2, 13, 3, 0.5, 4), (10, 3, 12, 2, 0.3, 3),
                                           (16, 2, 11, 2, 0.2, 4), (12, 2, 9, 2, 0.4, 9),
                                           (9, 1, 10, 2, 0.6, 2), (15, 4, 7, 2, 0.3, 5)])
def test_checkpoint_interval_gives_the_same_answer(B, L, k, n, N, T, C):
    (c, w, g), (w_hat, _, log_z, grad_w, grad_c) = _run_fwd_bwd(B, L, k, n, N, T, seed=5 + C, C=C)
    _, (w_hat1, _, log_z1, grad_w1, grad_c1) = _run_fwd_bwd(B, L, k, n, N, T, seed=5 + C, C=1)
    o_what, _, _ = oracle.forward(w, c, T, L, k)
    o_gw, o_gc = oracle.backward(g, w, c, T, L, k)
    assert_abs(w_hat, o_what, W_HAT_ATOL, "w_hat")
    assert_rel_l2(grad_w, o_gw, GRAD_REL_L2, "grad_w")
    assert_rel_l2(grad_c, o_gc, GRAD_REL_L2, "grad_codebook")
    # C > 1 runs another kernel instantiation (one sequence in flight per team,
    # the forward values recomputed per segment); the per-sequence outputs agree
    # to a few ulp, and grad_codebook sums the sequences in another order
    torch.testing.assert_close(log_z, log_z1, rtol=1e-6, atol=1e-6)
    torch.testing.assert_close(w_hat, w_hat1, rtol=0, atol=1e-6)
    torch.testing.assert_close(grad_w, grad_w1, rtol=1e-5, atol=1e-5)
    torch.testing.assert_close(grad_c, grad_c1, rtol=1e-5, atol=1e-5)


@pytest.mark.parametrize("L,k,n,N", [(8, 2, 64, 16), (4, 1, 7, 5), (6, 3, 9, 4), (9, 2, 12, 3), (12, 4, 10, 3),
                                       (14, 2, 12, 2), (15, 3, 10, 2), (16, 2, 9, 3), (16, 4, 7, 2)])
def test_viterbi_bit_exact(B, L, k, n, N):
    c, w, _ = _case(L, k, n, N, seed=40 + L + k)
    states, w_hard = B.viterbi_decode(w.cuda(), c.cuda(), L, k)
    o_states, o_hard, _ = oracle.viterbi(w, c, L, k)
    np.testing.assert_array_equal(states.cpu().numpy(), o_states)
    np.testing.assert_array_equal(w_hard.cpu().numpy(), o_hard)


def test_alternating_sizes_share_kernels(B):
    # L = 10 and L = 9 (k = 3) use the same kernel instantiation with different
    # shared-memory sizes; going back to the larger one must still launch.
    for L in (10, 9, 10, 9):
        (c, w, g), (w_hat, _, _, grad_w, _) = _run_fwd_bwd(B, L, 3, 6, 2, 0.4, seed=L)
        o_what, _, _ = oracle.forward(w, c, 0.4, L, 3)
        assert_abs(w_hat, o_what, W_HAT_ATOL, f"w_hat L={L}")


def test_single_step_and_empty_batch(B):
    L, k, T = 16, 2, 0.3
    (c, w, g), (w_hat, _, log_z, grad_w, grad_c) = _run_fwd_bwd(B, L, k, 1, 3, T, seed=77)
    o_what, o_lz, _ = oracle.forward(w, c, T, L, k)
    o_gw, o_gc = oracle.backward(g, w, c, T, L, k)
    assert_abs(w_hat, o_what, W_HAT_ATOL, "w_hat n=1")
    assert_rel_l2(grad_w, o_gw, GRAD_REL_L2, "grad_w n=1")
    assert_rel_l2(grad_c, o_gc, GRAD_REL_L2, "grad_c n=1")
    # N = 0: nothing to do; grad_codebook is cleared (not accumulated)
    w0 = torch.empty((0, 8), device="cuda")
    gc = torch.full((1 << L,), 7.0, device="cuda")
    B.bcjr_backward(w0, w0, c.cuda(), w0, T, L, k, grad_codebook=gc, accumulate_codebook=False)
    torch.cuda.synchronize()
    assert float(gc.abs().max()) == 0.0


def test_accumulate_codebook(B):
    L, k, n, N, T = 10, 2, 12, 3, 0.4
    c, w, g = _case(L, k, n, N, seed=88)
    dc, dw, dg = c.cuda(), w.cuda(), g.cuda()
    w_hat, _, _ = B.bcjr_forward(dw, dc, T, L, k)
    _, gc1 = B.bcjr_backward(dg, dw, dc, w_hat, T, L, k)
    acc = torch.ones(1 << L, device="cuda")
    B.bcjr_backward(dg, dw, dc, w_hat, T, L, k, grad_codebook=acc, accumulate_codebook=True)
    torch.cuda.synchronize()
    torch.testing.assert_close(acc, gc1 + 1.0, rtol=0, atol=1e-6)


def test_autograd_function(B):
    L, k, n, N, T = 9, 2, 10, 4, 0.5
    c, w, g = _case(L, k, n, N, seed=99)
    wv = w.cuda().requires_grad_(True)
    cv = c.cuda().requires_grad_(True)
    out = B.soft_quantize(wv, cv, T, L, k)
    (out * g.cuda()).sum().backward()
    o_gw, o_gc = oracle.backward(g, w, c, T, L, k)
    assert_rel_l2(wv.grad, o_gw, GRAD_REL_L2, "autograd grad_w")
    assert_rel_l2(cv.grad, o_gc, GRAD_REL_L2, "autograd grad_c")


def test_status_word_reports_non_finite_input(B):
    L, k, n, N, T = 10, 2, 6, 2, 0.5
    c, w, _ = _case(L, k, n, N, seed=5)
    w[1, 3] = float("nan")
    ws = B.Workspace("cuda")
    w_hat, _, _ = B.bcjr_forward(w.cuda(), c.cuda(), T, L, k, ws=ws)
    assert B.get_status(ws.buf) == 6
    w[1, 3] = 0.25
    B.bcjr_forward(w.cuda(), c.cuda(), T, L, k, ws=ws)
    assert B.get_status(ws.buf) == 0


def test_repeatable_bit_for_bit(B):
    L, k, n, N, T = 16, 2, 12, 5, 0.1
    _, a = _run_fwd_bwd(B, L, k, n, N, T, seed=3)
    _, b = _run_fwd_bwd(B, L, k, n, N, T, seed=3)
    for x, y in zip(a, b):
        if x is not None:
            assert torch.equal(x, y)
