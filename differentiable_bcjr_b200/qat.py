"""Per-layer reconstruction-MSE QAT on synthetic data.

"BCJR-QAT: A Differentiable Relaxation of Trellis-Coded Weight Quantization",
OLMoE experiment: greedy per-layer QAT that minimises the layer's
reconstruction mean squared error (a proxy objective), compared with the
hard-decoded post-training quantisation of the same weights.

Here: a layer W [R][C] (rows split into trellis sequences of `seq_len`
weights) and inputs X [B][C].  The preimage V starts at W; at each
temperature of an annealing schedule, a few optimiser steps minimise
mean((X W^T - X W_hat(V)^T)^2) with W_hat the BCJR soft codeword of V (the
library's forward and backward calls through autograd).  At the end V is
hard-decoded with the Viterbi call and compared with decoding W directly.
The matrix products are ordinary PyTorch; every trellis step runs in the
library's kernels.
"""
from __future__ import annotations

import torch

from . import soft_quantize, viterbi_decode


def _recon_mse(X, W_ref, W_q):
    return ((X @ (W_ref - W_q).T) ** 2).mean()


def layer_reconstruction_qat(W: torch.Tensor, X: torch.Tensor, codebook: torch.Tensor, state_bits: int, k: int,
                             seq_len: int, temperatures, steps_per_temperature: int = 10, lr: float = 0.02,
                             train_codebook: bool = False):
    """Returns a dict with the loss history, the hard-decoded reconstruction MSE
    after QAT (`mse_qat`), that of decoding W directly (`mse_ptq`), and the
    quantised weights."""
    if W.numel() % seq_len:
        raise ValueError("the layer must split into whole sequences")
    V = W.detach().clone().requires_grad_(True)
    cb = codebook.detach().clone().requires_grad_(train_codebook)
    params = [V] + ([cb] if train_codebook else [])
    opt = torch.optim.Adam(params, lr=lr)
    history = []
    for T in temperatures:
        for _ in range(steps_per_temperature):
            W_hat = soft_quantize(V.view(-1, seq_len), cb, float(T), state_bits, k).view_as(W)
            loss = _recon_mse(X, W, W_hat)
            opt.zero_grad(set_to_none=True)
            loss.backward()
            opt.step()
            history.append(loss.detach())
    with torch.no_grad():
        _, w_qat = viterbi_decode(V.detach().view(-1, seq_len).contiguous(), cb.detach(), state_bits, k)
        _, w_ptq = viterbi_decode(W.detach().view(-1, seq_len).contiguous(), codebook, state_bits, k)
        w_qat = w_qat.view_as(W)
        w_ptq = w_ptq.view_as(W)
        mse_qat = float(_recon_mse(X, W, w_qat))
        mse_ptq = float(_recon_mse(X, W, w_ptq))
    return {"history": [float(h) for h in history], "mse_qat": mse_qat, "mse_ptq": mse_ptq,
            "w_qat": w_qat, "w_ptq": w_ptq, "preimage": V.detach(), "codebook": cb.detach()}
