"""Sequence sharding over ranks (one process per GPU, torch.distributed).

The soft codeword is computed "for each independent weight sequence" (BCJR-QAT,
technical summary, "core mechanism": every row of the weight matrix is its own
trellis path), so the hot path shards by sequence with no exchange inside the
forward-backward: each rank owns a contiguous block of rows of w and runs
bcjr_forward / bcjr_backward on it.  The codebook is one table shared by every
sequence, so its gradient is summed over all rows; across ranks that is the
path's single collective, an all-reduce (sum) of S floats per backward call
(256 KiB at 2^16 states), over NCCL on GPUs.

Everything here is host-side bookkeeping around the library's calls; the
per-shard compute functions default to the CUDA library and can be replaced
(the multi-rank CPU tests pass their own).
"""
from __future__ import annotations

from typing import Callable, Optional, Tuple

import torch
import torch.distributed as dist

__all__ = ["shard_bounds", "local_rows", "all_reduce_codebook_grad", "max_over_ranks", "ShardedSoftQuant"]


def shard_bounds(n_seq: int, world_size: int, rank: int) -> Tuple[int, int]:
    """Rows [lo, hi) of an n_seq-row batch owned by `rank`: contiguous blocks
    whose sizes differ by at most one, the larger ones first."""
    if world_size < 1 or not 0 <= rank < world_size:
        raise ValueError(f"rank {rank} outside a world of {world_size}")
    if n_seq < 0:
        raise ValueError("n_seq must be >= 0")
    base, extra = divmod(n_seq, world_size)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def local_rows(t: torch.Tensor, world_size: int, rank: int) -> torch.Tensor:
    """This rank's block of rows of a [N][...] tensor (a view, no copy)."""
    lo, hi = shard_bounds(t.shape[0], world_size, rank)
    return t[lo:hi]


def all_reduce_codebook_grad(grad_codebook: torch.Tensor, group=None) -> torch.Tensor:
    """Sum the per-rank codebook gradients in place (no-op on one rank)."""
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(grad_codebook, op=dist.ReduceOp.SUM, group=group)
    return grad_codebook


def max_over_ranks(value: float, device=None, group=None) -> float:
    """The largest `value` over all ranks (device times are reported as the max)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size(group) == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())


Forward = Callable[..., Tuple[torch.Tensor, Optional[torch.Tensor], torch.Tensor]]
Backward = Callable[..., Tuple[torch.Tensor, torch.Tensor]]


class ShardedSoftQuant:
    """Forward and backward calls over this rank's sequences, with the codebook
    gradient summed over ranks.

        sq = ShardedSoftQuant(codebook, state_bits, k)
        w_hat = sq.forward(w_local, T)
        grad_w, grad_codebook = sq.backward(g_local, w_local, w_hat, T)

    `w_local` holds this rank's rows (see shard_bounds / local_rows).  The
    returned grad_codebook is the sum over every rank's sequences, identical on
    all ranks.  `forward_fn` / `backward_fn` default to the library's
    bcjr_forward / bcjr_backward and take the same arguments.
    """

    def __init__(self, codebook: torch.Tensor, state_bits: int, k: int, group=None,
                 forward_fn: Optional[Forward] = None, backward_fn: Optional[Backward] = None,
                 checkpoint_interval: int = 0, sequences_in_flight: int = 0):
        if forward_fn is None or backward_fn is None:
            from . import bcjr_backward, bcjr_forward
            forward_fn = forward_fn or bcjr_forward
            backward_fn = backward_fn or bcjr_backward
        self.codebook = codebook
        self.state_bits = int(state_bits)
        self.k = int(k)
        self.group = group
        self.C = int(checkpoint_interval)
        self.fwd_kw = {"sequences_in_flight": int(sequences_in_flight)} if sequences_in_flight else {}
        self._fwd = forward_fn
        self._bwd = backward_fn
        self._grad_c = None

    def forward(self, w_local: torch.Tensor, T: float, out: Optional[torch.Tensor] = None) -> torch.Tensor:
        w_hat, _, _ = self._fwd(w_local, self.codebook, T, self.state_bits, self.k,
                                checkpoint_interval=self.C, out=out, **self.fwd_kw)
        return w_hat

    def backward(self, g_local: torch.Tensor, w_local: torch.Tensor, w_hat_local: torch.Tensor,
                 T: float) -> Tuple[torch.Tensor, torch.Tensor]:
        S = 1 << self.state_bits
        if self._grad_c is None or self._grad_c.device != self.codebook.device:
            self._grad_c = torch.zeros(S, dtype=torch.float32, device=self.codebook.device)
        grad_w, grad_c = self._bwd(g_local, w_local, self.codebook, w_hat_local, T, self.state_bits, self.k,
                                   checkpoint_interval=self.C, grad_codebook=self._grad_c,
                                   accumulate_codebook=False)
        all_reduce_codebook_grad(grad_c, self.group)
        return grad_w, grad_c
