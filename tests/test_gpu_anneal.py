"""The captured annealing sweep against the same calls made one by one, and
against the oracle (needs a B200)."""
import numpy as np
import pytest
import torch

import bcjr_inputs as I
import oracle
from parity import GRAD_REL_L2, W_HAT_ATOL, assert_abs, assert_rel_l2

pytestmark = pytest.mark.gpu


def test_graph_replay_matches_eager_calls_and_the_oracle():
    import differentiable_bcjr_b200 as B
    from differentiable_bcjr_b200.anneal import AnnealSweep
    L, k, n, N = 10, 2, 24, 37
    temps = I.anneal_temperatures(0.3, 0.01, 3)
    c = I.codebook(1 << L, seed=61).cuda()
    sweep = AnnealSweep(c, temps, L, k, N, n)
    for rep in range(2):  # two replays on different inputs
        w = I.weights(N, n, seed=62 + rep).cuda()
        g = I.upstream_grad(N, n, seed=63 + rep).cuda()
        w_hat, grad_w, grad_c = sweep.run(w, g)
        torch.cuda.synchronize()
        for i, T in enumerate(temps):
            e_what, _, _ = B.bcjr_forward(w, c, T, L, k)
            e_gw, e_gc = B.bcjr_backward(g, w, c, e_what, T, L, k)
            torch.cuda.synchronize()
            assert torch.equal(w_hat[i], e_what) and torch.equal(grad_w[i], e_gw) and torch.equal(grad_c[i], e_gc)
        o_what, _, _ = oracle.forward(w.cpu(), c.cpu(), temps[-1], L, k)
        o_gw, o_gc = oracle.backward(g.cpu(), w.cpu(), c.cpu(), temps[-1], L, k)
        assert_abs(w_hat[-1], o_what, W_HAT_ATOL, "w_hat at the last temperature")
        assert_rel_l2(grad_w[-1], o_gw, GRAD_REL_L2, "grad_w at the last temperature")
        assert_rel_l2(grad_c[-1], o_gc, GRAD_REL_L2, "grad_codebook at the last temperature")


def test_graph_replay_on_a_cluster_team():
    # state_bits = 16: 8-CTA clusters, st.async exchange and mbarriers inside the graph
    from differentiable_bcjr_b200.anneal import AnnealSweep
    import differentiable_bcjr_b200 as B
    L, k, n, N = 16, 2, 12, 5
    temps = [0.3, 0.05]
    c = I.codebook(1 << L).cuda()
    w, g = I.weights(N, n).cuda(), I.upstream_grad(N, n).cuda()
    sweep = AnnealSweep(c, temps, L, k, N, n)
    w_hat, grad_w, grad_c = sweep.run(w, g)
    torch.cuda.synchronize()
    e_what, _, _ = B.bcjr_forward(w, c, temps[1], L, k)
    e_gw, e_gc = B.bcjr_backward(g, w, c, e_what, temps[1], L, k)
    torch.cuda.synchronize()
    assert torch.equal(w_hat[1], e_what) and torch.equal(grad_w[1], e_gw) and torch.equal(grad_c[1], e_gc)
    assert np.isfinite(grad_c.cpu().numpy()).all()
