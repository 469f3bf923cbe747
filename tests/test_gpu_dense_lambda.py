"""GPU parity of the log-transition gradient of the dense trellis (needs a B200).

bcjr_dense_backward_lambda returns dL/dLambda next to the usual VJP; the sum
over (sequence, transition) rows runs on the tcgen05 tensor cores in
three-pass tf32.  Checked against the float64 oracle (itself pinned to path
enumeration and finite differences) at lengths 1 (no transitions: zero), 2, 7
and 64, batches that fill one tile, leave a ragged tail and span several tiles;
against the zero-sum invariant (a common shift of Lambda changes no path's
probability); and, for a batch longer than one launch, against the sum of the
two halves computed separately.
"""
import numpy as np
import pytest
import torch

import bcjr_inputs as I
import oracle
from parity import GRAD_REL_L2, assert_rel_l2, to_np

pytestmark = pytest.mark.gpu

S = 256


@pytest.fixture(scope="module")
def B():
    import differentiable_bcjr_b200 as B
    B.lib()
    return B


def _case(n, N, seed):
    return (I.codebook(S, seed=500 + seed), I.weights(N, n, seed=600 + seed), I.upstream_grad(N, n, seed=700 + seed),
            I.log_transition(S, seed=800 + seed))


@pytest.mark.parametrize("n,N,T", [(1, 3, 0.5), (2, 5, 0.7), (7, 40, 0.2), (64, 40, 1.0), (64, 70, 0.2),
                                   (16, 33, 0.02)])
def test_log_transition_gradient_parity(B, n, N, T):
    c, w, g, lam = _case(n, N, seed=n + N)
    dc, dw, dg, dl = c.cuda(), w.cuda(), g.cuda(), lam.cuda()
    w_hat, _, _ = B.bcjr_dense_forward(dw, dc, dl, T)
    gw, gc, gl = B.bcjr_dense_backward(dg, dw, dc, dl, w_hat, T, want_grad_log_trans=True)
    gw0, gc0 = B.bcjr_dense_backward(dg, dw, dc, dl, w_hat, T)
    torch.cuda.synchronize()
    # the extra output changes nothing in the others (one launch: the same
    # kernel, tiles and reduction order as the plain call)
    assert torch.equal(gw, gw0)
    assert torch.equal(gc, gc0)
    o_gw, o_gc, o_gl = oracle.dense_backward(g, w, c, lam, T, want_grad_lam=True)
    assert_rel_l2(gw0, o_gw, GRAD_REL_L2, "grad_w (plain call)")
    assert_rel_l2(gc0, o_gc, GRAD_REL_L2, "grad_codebook (plain call)")
    if n == 1:
        assert bool((gl == 0).all())
        return
    err = float(np.linalg.norm(to_np(gl) - o_gl) / np.linalg.norm(o_gl))
    print(f"grad_log_trans rel L2 {err:.3e}")
    assert_rel_l2(gl, o_gl, GRAD_REL_L2, "grad_log_trans")
    # float32-level accuracy is the design (three-pass tf32); one-pass tf32
    # would sit near 5e-4, so hold the result well below that
    assert err < 2e-5, err
    assert_rel_l2(gw, o_gw, GRAD_REL_L2, "grad_w")


def test_log_transition_gradient_sums_to_zero_and_repeats(B):
    n, N, T = 33, 300, 0.25
    c, w, g, lam = _case(n, N, seed=3)
    dc, dw, dg, dl = c.cuda(), w.cuda(), g.cuda(), lam.cuda()
    w_hat, _, _ = B.bcjr_dense_forward(dw, dc, dl, T)
    _, _, a = B.bcjr_dense_backward(dg, dw, dc, dl, w_hat, T, want_grad_log_trans=True)
    _, _, b = B.bcjr_dense_backward(dg, dw, dc, dl, w_hat, T, want_grad_log_trans=True)
    torch.cuda.synchronize()
    assert torch.equal(a, b)  # fixed-order reduction: run-to-run identical
    x = a.double()
    assert abs(float(x.sum())) <= 1e-5 * float(x.abs().sum())
    assert float(x.abs().max()) > 0


def test_log_transition_gradient_over_several_launches(B):
    # More sequences than one launch holds (one 64-sequence tile per resident
    # cluster): the call runs in chunks and accumulates; compare with the two
    # halves computed apart.
    B.lib()
    n, T = 3, 0.4
    import ctypes
    o = B._opts(0)
    # find the chunk length: the smallest N whose workspace stops growing with N
    chunk = None
    prev = B.lib().bcjr_workspace_size(B.OP_DENSE_BACKWARD_LAMBDA, 8, 0, n, 32, ctypes.byref(o))
    for N in range(64, 32 * 1024 + 1, 32):
        cur = B.lib().bcjr_workspace_size(B.OP_DENSE_BACKWARD_LAMBDA, 8, 0, n, N, ctypes.byref(o))
        if cur == prev:
            chunk = N - 32
            break
        prev = cur
    assert chunk is not None and chunk % 32 == 0
    N = chunk + 40
    c, w, g, lam = _case(n, N, seed=4)
    dc, dw, dg, dl = c.cuda(), w.cuda(), g.cuda(), lam.cuda()
    w_hat, _, _ = B.bcjr_dense_forward(dw, dc, dl, T)
    gw, gc, gl = B.bcjr_dense_backward(dg, dw, dc, dl, w_hat, T, want_grad_log_trans=True)
    parts = []
    for sl in (slice(0, chunk), slice(chunk, N)):
        parts.append(B.bcjr_dense_backward(dg[sl].contiguous(), dw[sl].contiguous(), dc, dl,
                                           w_hat[sl].contiguous(), T, want_grad_log_trans=True))
    torch.cuda.synchronize()
    assert torch.equal(gw, torch.cat([parts[0][0], parts[1][0]]))
    ref_c = (parts[0][1].double() + parts[1][1].double())
    ref_l = (parts[0][2].double() + parts[1][2].double())
    assert float((gc.double() - ref_c).norm() / ref_c.norm()) < 1e-6
    assert float((gl.double() - ref_l).norm() / ref_l.norm()) < 1e-6


def test_dense_autograd_function(B):
    n, N, T = 12, 35, 0.3
    c, w, g, lam = _case(n, N, seed=5)
    wv = w.cuda().requires_grad_(True)
    cv = c.cuda().requires_grad_(True)
    lv = lam.cuda().requires_grad_(True)
    w_hat = B.dense_soft_quantize(wv, cv, lv, T)
    (w_hat * g.cuda()).sum().backward()
    o_gw, o_gc, o_gl = oracle.dense_backward(g, w, c, lam, T, want_grad_lam=True)
    assert_rel_l2(wv.grad, o_gw, GRAD_REL_L2, "grad_w")
    assert_rel_l2(cv.grad, o_gc, GRAD_REL_L2, "grad_c")
    assert_rel_l2(lv.grad, o_gl, GRAD_REL_L2, "grad_log_trans")
    # without a log_trans gradient the plain backward call runs
    lv2 = lam.cuda()
    w2 = w.cuda().requires_grad_(True)
    (B.dense_soft_quantize(w2, c.cuda(), lv2, T) * g.cuda()).sum().backward()
    assert torch.equal(w2.grad, wv.grad)


@pytest.mark.slow
def test_log_transition_gradient_full_workload(B):
    # 4096 sequences x 4096 steps (the dense workload): the oracle cannot run
    # at this size, so check what holds at any size -- the zero sum, agreement
    # of the other outputs with the plain backward call (grad_w bit for bit;
    # grad_codebook to float32 rounding, since this call runs the tiles in two
    # launches and adds their codebook partials in another order), run-to-run
    # identity.
    W = I.WORKLOADS["dense_S256"]
    n, N, T = W["seq_len"], W["n_seq"], W["T"][0]
    c, w, g, lam = I.codebook(S).cuda(), I.weights(N, n).cuda(), I.upstream_grad(N, n).cuda(), I.log_transition(S).cuda()
    w_hat, _, _ = B.bcjr_dense_forward(w, c, lam, T)
    gw, gc, gl = B.bcjr_dense_backward(g, w, c, lam, w_hat, T, want_grad_log_trans=True)
    gw0, gc0 = B.bcjr_dense_backward(g, w, c, lam, w_hat, T)
    _, _, gl2 = B.bcjr_dense_backward(g, w, c, lam, w_hat, T, want_grad_log_trans=True)
    torch.cuda.synchronize()
    assert torch.equal(gw, gw0)
    assert_rel_l2(gc, to_np(gc0), 1e-5, "grad_codebook of the two calls")
    assert torch.equal(gl, gl2)
    x = gl.double()
    assert bool(torch.isfinite(x).all())
    # Each CTA accumulates about N (n-1) / 148 = 113k rows (6 tf32 products
    # per row pair, float32 accumulator), so rounding leaves each entry a
    # random-walk error near sqrt(6 * 113k) * 2^-24 ~ 5e-5 of its size.  The
    # exact sum is zero; allow ten times that walk.
    assert abs(float(x.sum())) <= 5e-4 * float(x.abs().sum())


def test_log_transition_gradient_accumulates(B):
    n, N, T = 9, 37, 0.35
    c, w, g, lam = _case(n, N, seed=6)
    dc, dw, dg, dl = c.cuda(), w.cuda(), g.cuda(), lam.cuda()
    w_hat, _, _ = B.bcjr_dense_forward(dw, dc, dl, T)
    _, gc1, gl1 = B.bcjr_dense_backward(dg, dw, dc, dl, w_hat, T, want_grad_log_trans=True)
    gc = torch.full((S,), 0.25, device="cuda")
    gl = torch.full((S, S), -0.5, device="cuda")
    B.bcjr_dense_backward(dg, dw, dc, dl, w_hat, T, want_grad_log_trans=True, grad_codebook=gc,
                          grad_log_trans=gl, accumulate=True)
    torch.cuda.synchronize()
    torch.testing.assert_close(gc, gc1 + 0.25, rtol=0, atol=1e-6)
    torch.testing.assert_close(gl, gl1 - 0.5, rtol=0, atol=1e-6)


def test_log_transition_gradient_empty_batch(B):
    c, _, _, lam = _case(5, 1, seed=7)
    w0 = torch.empty((0, 5), device="cuda")
    gw, gc, gl = B.bcjr_dense_backward(w0, w0, c.cuda(), lam.cuda(), w0, 0.3, want_grad_log_trans=True)
    torch.cuda.synchronize()
    assert gw.numel() == 0 and bool((gc == 0).all()) and bool((gl == 0).all())
