"""Seeded synthetic inputs for BCJR-QAT workloads.

Shared by the tests, the benchmark and the smoke check; used by both the CUDA
path and the float64 oracle, so it holds no forward-backward arithmetic: it
only draws the numbers.  Every tensor is drawn on the CPU from
``torch.Generator().manual_seed(seed)`` as float32, so the same bits go to the
GPU and to the oracle.

Workloads (stand-ins for the paper's Hadamard-incoherent LLM weights, which
are not available here): weights, codebook, upstream gradient and the dense
log-transition matrix are all iid N(0, 1).
"""
from __future__ import annotations

import math

import torch

SEED_CODEBOOK = 0
SEED_WEIGHTS = 1
SEED_UPSTREAM = 2
SEED_TRANSITION = 3


def normal(shape, seed: int) -> torch.Tensor:
    """iid N(0, 1) float32 on the CPU from a fixed seed."""
    g = torch.Generator().manual_seed(int(seed))
    return torch.randn(*shape, generator=g, dtype=torch.float32)


def codebook(n_states: int, seed: int = SEED_CODEBOOK) -> torch.Tensor:
    """One scalar codeword per trellis state: [S] float32."""
    return normal((n_states,), seed)


def weights(n_seq: int, seq_len: int, seed: int = SEED_WEIGHTS) -> torch.Tensor:
    """Weight sequences [N][n] float32.  A projection matrix of R x C weights
    viewed row-major as [R*C/n][n] has exactly these bits when drawn with the
    same seed, so "a 2048 x 8192 matrix split into 65536 rows of 256" is
    weights(65536, 256)."""
    return normal((n_seq, seq_len), seed)


def upstream_grad(n_seq: int, seq_len: int, seed: int = SEED_UPSTREAM) -> torch.Tensor:
    """Upstream gradient dL/dw_hat [N][n] float32."""
    return normal((n_seq, seq_len), seed)


def log_transition(n_states: int, seed: int = SEED_TRANSITION) -> torch.Tensor:
    """Dense log-transition matrix [S][S] float32: iid N(0, 1) entries, each
    row shifted so that its exponentials sum to one (row = source state).
    The shift is taken in float64 and the result rounded once to float32."""
    raw = normal((n_states, n_states), seed).double()
    return (raw - torch.logsumexp(raw, dim=1, keepdim=True)).float()


def anneal_temperatures(t0: float = 0.3, t_end: float = 0.005, steps: int = 8) -> list[float]:
    """Geometric annealing schedule T_i = t0 * (t_end / t0) ** (i / (steps - 1))."""
    if steps == 1:
        return [float(t0)]
    return [float(t0 * (t_end / t0) ** (i / (steps - 1))) for i in range(steps)]


# The five workloads, by what they are.  "T" lists every temperature run.
WORKLOADS = {
    "tiny_L8_k2": dict(state_bits=8, k=2, seq_len=64, n_seq=16, T=[0.5]),
    "qtip_L16_k2_n16": dict(state_bits=16, k=2, seq_len=256, n_seq=16, T=[1.0, 0.3, 0.1, 0.01]),
    "proj2048x8192_L16_k2": dict(state_bits=16, k=2, seq_len=256, n_seq=65536,
                                 T=anneal_temperatures(0.3, 0.005, 8)),
    "bitwidth_L16_k234": dict(state_bits=16, k=[2, 3, 4], seq_len=256, n_seq=16384, T=[0.1]),
    "dense_S256": dict(n_states=256, seq_len=4096, n_seq=4096, T=[0.2]),
}

LN2 = math.log(2.0)
