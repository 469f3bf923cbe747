"""Element-wise parity on 256-sequence subsets of the two large workloads
(needs a B200).

The first 256 rows of the 2048 x 8192 projection (2^16 states, k = 2) at the
first and last temperature of its annealing sweep, and of the bit-width sweep
at k = 3 and k = 4 (T = 0.1), go through the same entry points as a
256-sequence call; w_hat, log Z, grad_w and grad_codebook (summed over the 256
sequences) are compared with the float64 oracle's values, which
tests/golden/make_subset_parity.py wrote from the oracle alone (they take
about 40 CPU-minutes, too long to recompute inside every GPU run).
"""
import os

import numpy as np
import pytest
import torch

import bcjr_inputs as I
from parity import (GRAD_REL_L2, LOGZ_ATOL_PER_STEP, LOGZ_RTOL, W_HAT_ATOL, assert_abs, assert_rel_l2,
                    to_np)

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
CASES = ["proj_T0", "proj_T7", "bitwidth_k3", "bitwidth_k4"]


@pytest.mark.parametrize("name", CASES)
def test_subset_matches_the_oracle(name):
    import differentiable_bcjr_b200 as B
    ref = np.load(os.path.join(GOLDEN, f"subset_{name}.npz"))
    L, k, n, T, N = int(ref["L"]), int(ref["k"]), int(ref["n"]), float(ref["T"]), int(ref["n_seq"])
    dev = torch.device("cuda", 0)
    c, w, g = I.codebook(1 << L).to(dev), I.weights(N, n).to(dev), I.upstream_grad(N, n).to(dev)
    w_hat, _, log_z = B.bcjr_forward(w, c, T, L, k)
    grad_w, grad_c = B.bcjr_backward(g, w, c, w_hat, T, L, k)
    torch.cuda.synchronize()
    assert_abs(w_hat, ref["w_hat"], W_HAT_ATOL, f"{name} w_hat")
    np.testing.assert_allclose(to_np(log_z), ref["log_z"], rtol=LOGZ_RTOL, atol=LOGZ_ATOL_PER_STEP * n)
    assert_rel_l2(grad_w, ref["grad_w"], GRAD_REL_L2, f"{name} grad_w")
    assert_rel_l2(grad_c, ref["grad_codebook"], GRAD_REL_L2, f"{name} grad_codebook")
