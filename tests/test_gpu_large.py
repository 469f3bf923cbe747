"""Full-size workloads on the GPU, checked against the oracle (needs a B200).

  * QTIP-scale trellis, L=16 (S=65536), k=2, 256 steps, 16 sequences:
    every sequence vs the oracle, forward and backward at T in
    {1, 0.3, 0.1, 0.01}, hard decode bit-exact;
  * the 2048 x 8192 projection matrix as 65536 sequences of 256 (the
    benchmark's launch): sampled sequences vs the oracle one by one at the
    first and last temperature of the annealing sweep, plus the translation
    identity sum grad_w + sum grad_codebook = sum g over all 16.7M weights;
    its hard decode: sampled sequences bit-exact, codewords and transitions
    valid everywhere;
  * the bit-width sweep, k = 3 and 4 on 16384 sequences: sampled sequences
    and the translation identity.
"""
import numpy as np
import pytest
import torch

import bcjr_inputs as I
import oracle
from parity import (GRAD_REL_L2, LOGZ_ATOL_PER_STEP, LOGZ_RTOL, W_HAT_ATOL, assert_abs, assert_rel_l2,
                    to_np)

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module")
def B():
    import differentiable_bcjr_b200 as B
    B.lib()
    return B


@pytest.fixture(scope="module")
def qtip_inputs():
    W = I.WORKLOADS["qtip_L16_k2_n16"]
    L, k, n, N = W["state_bits"], W["k"], W["seq_len"], W["n_seq"]
    return L, k, I.codebook(1 << L), I.weights(N, n), I.upstream_grad(N, n)


@pytest.mark.parametrize("T", [1.0, 0.3, 0.1, 0.01])
def test_qtip_scale_forward(B, qtip_inputs, T):
    L, k, c, w, _ = qtip_inputs
    w_hat, _, log_z = B.bcjr_forward(w.cuda(), c.cuda(), T, L, k)
    o_what, o_lz, _ = oracle.forward(w, c, T, L, k)
    assert_abs(w_hat, o_what, W_HAT_ATOL, f"w_hat T={T}")
    np.testing.assert_allclose(to_np(log_z), o_lz, rtol=LOGZ_RTOL, atol=LOGZ_ATOL_PER_STEP * w.shape[1])


@pytest.mark.parametrize("T", [1.0, 0.3, 0.1, 0.01])
def test_qtip_scale_backward(B, qtip_inputs, T):
    L, k, c, w, g = qtip_inputs
    dw, dc = w.cuda(), c.cuda()
    w_hat, _, _ = B.bcjr_forward(dw, dc, T, L, k)
    grad_w, grad_c = B.bcjr_backward(g.cuda(), dw, dc, w_hat, T, L, k)
    o_gw, o_gc = oracle.backward(g, w, c, T, L, k)
    assert_rel_l2(grad_w, o_gw, GRAD_REL_L2, f"grad_w T={T}")
    assert_rel_l2(grad_c, o_gc, GRAD_REL_L2, f"grad_codebook T={T}")


def test_qtip_scale_viterbi(B, qtip_inputs):
    L, k, c, w, _ = qtip_inputs
    states, w_hard = B.viterbi_decode(w.cuda(), c.cuda(), L, k)
    o_states, o_hard, _ = oracle.viterbi(w, c, L, k)
    np.testing.assert_array_equal(states.cpu().numpy(), o_states)
    np.testing.assert_array_equal(w_hard.cpu().numpy(), o_hard)


def _translation_identity(grad_w, grad_c, g):
    lhs = grad_w.double().sum().item() + grad_c.double().sum().item()
    rhs = g.double().sum().item()
    scale = grad_w.double().abs().sum().item() + grad_c.double().abs().sum().item()
    assert abs(lhs - rhs) <= 1e-4 * scale, (lhs, rhs, scale)


@pytest.mark.parametrize("T", [I.anneal_temperatures()[0], I.anneal_temperatures()[-1]])
def test_projection_matrix_sampled(B, T):
    W = I.WORKLOADS["proj2048x8192_L16_k2"]
    L, k, n, N = W["state_bits"], W["k"], W["seq_len"], W["n_seq"]
    c, w, g = I.codebook(1 << L), I.weights(N, n), I.upstream_grad(N, n)
    dw, dc, dg = w.cuda(), c.cuda(), g.cuda()
    w_hat, _, _ = B.bcjr_forward(dw, dc, T, L, k)
    grad_w, grad_c = B.bcjr_backward(dg, dw, dc, w_hat, T, L, k)
    torch.cuda.synchronize()
    sample = [0, 1, 31337, N - 1]
    o_what, _, _ = oracle.forward(w[sample], c, T, L, k)
    o_gw, _ = oracle.backward(g[sample], w[sample], c, T, L, k)
    assert_abs(w_hat[sample], o_what, W_HAT_ATOL, f"w_hat sampled T={T}")
    assert_rel_l2(grad_w[sample], o_gw, GRAD_REL_L2, f"grad_w sampled T={T}")
    _translation_identity(grad_w, grad_c, g)


@pytest.mark.parametrize("k", [3, 4])
def test_bitwidth_sweep_sampled(B, k):
    W = I.WORKLOADS["bitwidth_L16_k234"]
    L, n, N, T = W["state_bits"], W["seq_len"], W["n_seq"], W["T"][0]
    c, w, g = I.codebook(1 << L), I.weights(N, n), I.upstream_grad(N, n)
    dw, dc, dg = w.cuda(), c.cuda(), g.cuda()
    w_hat, _, _ = B.bcjr_forward(dw, dc, T, L, k)
    grad_w, grad_c = B.bcjr_backward(dg, dw, dc, w_hat, T, L, k)
    torch.cuda.synchronize()
    sample = [0, N // 2 + 3, N - 1]
    o_what, _, _ = oracle.forward(w[sample], c, T, L, k)
    o_gw, _ = oracle.backward(g[sample], w[sample], c, T, L, k)
    assert_abs(w_hat[sample], o_what, W_HAT_ATOL, f"w_hat k={k}")
    assert_rel_l2(grad_w[sample], o_gw, GRAD_REL_L2, f"grad_w k={k}")
    _translation_identity(grad_w, grad_c, g)


def test_projection_hard_decode_sampled(B):
    # The hard-decode launch the benchmark times (65536 sequences): sampled
    # sequences bit-exact against the oracle's max-sum, and every decoded
    # codeword equal to the codebook entry of its state.
    W = I.WORKLOADS["proj2048x8192_L16_k2"]
    L, k, n, N = W["state_bits"], W["k"], W["seq_len"], W["n_seq"]
    c, w = I.codebook(1 << L), I.weights(N, n)
    dc = c.cuda()
    states, w_hard = B.viterbi_decode(w.cuda(), dc, L, k)
    torch.cuda.synchronize()
    sample = [0, 1, 4097, 31337, N - 2, N - 1]
    o_states = oracle.viterbi(w[sample], c, L, k)[0]
    assert (to_np(states[sample]) == o_states).all()
    assert torch.equal(w_hard, dc[states.long()])
    # every consecutive pair of states is a trellis transition
    s = states.long()
    assert bool(((s[:, 1:] >> k) == (s[:, :-1] & ((1 << (L - k)) - 1))).all())
