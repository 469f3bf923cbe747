"""GPU parity of the dense-trellis calls with the float64 oracle (needs a B200).

Shapes: 256 states (the size the kernels are built for); sequence counts
against the cluster tiles (128 sequences in the soft-codeword call, 64 in the
vector-Jacobian product): part of one tile (3, 40), a tile plus a ragged
rest (70, 129), several tiles (300, 2100), and more tiles than the 33
clusters that fit at once in both calls (4300: 34 and 68 tiles, so clusters
run several tiles in turn); lengths 1 (a plain softmax per sequence), 2, 3,
7, 16, 33 and 64; several temperatures.  The
full dense workload (4096 sequences of 4096 steps) is checked on sampled
sequences and by the translation identity.
"""
import numpy as np
import pytest
import torch

import bcjr_inputs as I
import oracle
from parity import (GRAD_REL_L2, LOGZ_ATOL_PER_STEP, LOGZ_RTOL, MARGINAL_ATOL, W_HAT_ATOL, assert_abs,
                    assert_rel_l2, to_np)

pytestmark = pytest.mark.gpu

S = 256


@pytest.fixture(scope="module")
def B():
    import differentiable_bcjr_b200 as B
    B.lib()
    return B


def _case(n, N, seed):
    return (I.codebook(S, seed=100 + seed), I.weights(N, n, seed=200 + seed), I.upstream_grad(N, n, seed=300 + seed),
            I.log_transition(S, seed=400 + seed))


@pytest.mark.parametrize("n,N,T", [(1, 3, 0.5), (7, 40, 0.2), (64, 40, 1.0), (64, 70, 0.2), (2, 129, 0.3),
                                   (33, 300, 0.2), (16, 2100, 0.5), (3, 4300, 0.3)])
def test_dense_parity(B, n, N, T):
    c, w, g, lam = _case(n, N, seed=n + N)
    dc, dw, dg, dl = c.cuda(), w.cuda(), g.cuda(), lam.cuda()
    w_hat, marg, log_z = B.bcjr_dense_forward(dw, dc, dl, T, want_marginals=True)
    grad_w, grad_c = B.bcjr_dense_backward(dg, dw, dc, dl, w_hat, T)
    torch.cuda.synchronize()
    o_what, o_lz, o_gamma = oracle.dense_forward(w, c, lam, T, want_gamma=True)
    o_gw, o_gc = oracle.dense_backward(g, w, c, lam, T)
    assert_abs(w_hat, o_what, W_HAT_ATOL, "w_hat")
    assert_abs(marg, o_gamma, MARGINAL_ATOL, "marginals")
    np.testing.assert_allclose(to_np(log_z), o_lz, rtol=LOGZ_RTOL, atol=LOGZ_ATOL_PER_STEP * n)
    assert_rel_l2(grad_w, o_gw, GRAD_REL_L2, "grad_w")
    assert_rel_l2(grad_c, o_gc, GRAD_REL_L2, "grad_c")
    # translation identity: shifting w and c together leaves every distance unchanged
    gsum = float(g.double().sum())
    tot = float(to_np(grad_w).sum() + to_np(grad_c).sum())
    assert abs(tot - gsum) <= 1e-4 * max(1.0, abs(gsum))


def test_dense_empty_batch_and_repeatability(B):
    c, w, g, lam = _case(9, 33, seed=1)
    dc, dw, dg, dl = c.cuda(), w.cuda(), g.cuda(), lam.cuda()
    a = B.bcjr_dense_forward(dw, dc, dl, 0.3)
    b = B.bcjr_dense_forward(dw, dc, dl, 0.3)
    assert torch.equal(a[0], b[0]) and torch.equal(a[2], b[2])
    ga = B.bcjr_dense_backward(dg, dw, dc, dl, a[0], 0.3)
    gb = B.bcjr_dense_backward(dg, dw, dc, dl, a[0], 0.3)
    assert torch.equal(ga[0], gb[0]) and torch.equal(ga[1], gb[1])
    w0 = torch.empty((0, 9), device="cuda")
    gw0, gc0 = B.bcjr_dense_backward(w0, w0, dc, dl, w0, 0.3)
    torch.cuda.synchronize()
    assert gw0.numel() == 0 and bool((gc0 == 0).all())


@pytest.mark.slow
def test_dense_full_workload_sampled(B):
    W = I.WORKLOADS["dense_S256"]
    n, N, T = W["seq_len"], W["n_seq"], W["T"][0]
    c, w, g, lam = I.codebook(S), I.weights(N, n), I.upstream_grad(N, n), I.log_transition(S)
    dc, dw, dg, dl = c.cuda(), w.cuda(), g.cuda(), lam.cuda()
    w_hat, _, log_z = B.bcjr_dense_forward(dw, dc, dl, T)
    grad_w, grad_c = B.bcjr_dense_backward(dg, dw, dc, dl, w_hat, T)
    torch.cuda.synchronize()
    rows = [0, 1, N - 1]
    o_what, o_lz, _ = oracle.dense_forward(w[rows], c, lam, T)
    o_gw, _ = oracle.dense_backward(g[rows], w[rows], c, lam, T)
    assert_abs(w_hat[rows], o_what, W_HAT_ATOL, "w_hat (sampled rows)")
    np.testing.assert_allclose(to_np(log_z[rows]), o_lz, rtol=LOGZ_RTOL, atol=LOGZ_ATOL_PER_STEP * n)
    assert_rel_l2(grad_w[rows], o_gw, GRAD_REL_L2, "grad_w (sampled rows)")
    gsum = float(g.double().sum())
    tot = float(to_np(grad_w).sum() + to_np(grad_c).sum())
    assert abs(tot - gsum) <= 1e-4 * max(1.0, abs(gsum)) + 1e-6 * float(to_np(grad_c).__abs__().sum())
