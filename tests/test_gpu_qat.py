"""Synthetic per-layer reconstruction QAT through the library (needs a B200)."""
import math

import pytest
import torch

import bcjr_inputs as I

pytestmark = pytest.mark.gpu


def test_layer_qat_lowers_the_reconstruction_error():
    from differentiable_bcjr_b200.qat import layer_reconstruction_qat
    L, k, n = 8, 2, 64
    R, C, Bsz = 16, 256, 128
    W = I.normal((R, C), seed=71).cuda()
    X = I.normal((Bsz, C), seed=72).cuda()
    c = I.codebook(1 << L, seed=73).cuda()
    steps = 8
    res = layer_reconstruction_qat(W, X, c, L, k, n, I.anneal_temperatures(0.3, 0.01, 4),
                                   steps_per_temperature=steps, lr=0.02)
    h = res["history"]
    assert all(math.isfinite(v) for v in h)
    # at the warmest temperature the soft objective goes down step by step (it rises
    # between temperatures: a colder soft codeword is closer to the hard code, and the
    # colder landscapes are rougher)
    assert all(b < a for a, b in zip(h[:steps], h[1:steps]))
    assert math.isfinite(res["mse_qat"]) and math.isfinite(res["mse_ptq"])
    assert res["mse_qat"] < res["mse_ptq"]            # QAT beats decoding the weights directly
    # the hard code is a path of the trellis: every value is a codeword
    cb = set(c.cpu().tolist())
    assert set(res["w_qat"].flatten().cpu().tolist()) <= cb
