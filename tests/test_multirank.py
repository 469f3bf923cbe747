"""Multi-rank sequence sharding on CPU (gloo ranks, no GPU).

Drives the package's sharding module (differentiable_bcjr_b200.distributed)
with per-shard compute functions built on the float64 oracle: every rank owns
a contiguous block of sequences, and the one cross-rank exchange is the
all-reduce (sum) of grad_codebook.  The sharded results must equal the
single-process results of the whole batch, for two and three ranks and for a
batch smaller than the world (a rank with no sequences).
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bcjr_inputs as I
import oracle
from differentiable_bcjr_b200 import distributed as D

L, K_BITS, SEQ_LEN, T = 6, 2, 5, 0.4


def _oracle_forward(w, c, T, L, k, checkpoint_interval=0, out=None):
    w_hat, log_z, _ = oracle.forward(w, c, T, L, k, nthreads=1)
    return torch.from_numpy(w_hat), None, torch.from_numpy(log_z)


def _oracle_backward(g, w, c, w_hat, T, L, k, checkpoint_interval=0, grad_codebook=None,
                     accumulate_codebook=False):
    gw, gc = oracle.backward(g, w, c, T, L, k, nthreads=1)
    grad_codebook.copy_(torch.from_numpy(gc).float())
    return torch.from_numpy(gw), grad_codebook


def _worker(rank, world, port, n_seq, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        c = I.codebook(1 << L, seed=11)
        w = I.weights(n_seq, SEQ_LEN, seed=12)
        g = I.upstream_grad(n_seq, SEQ_LEN, seed=13)
        lo, hi = D.shard_bounds(n_seq, world, rank)
        w_loc, g_loc = D.local_rows(w, world, rank), D.local_rows(g, world, rank)
        sq = D.ShardedSoftQuant(c, L, K_BITS, forward_fn=_oracle_forward, backward_fn=_oracle_backward)
        w_hat = sq.forward(w_loc, T)
        gw, gc = sq.backward(g_loc, w_loc, w_hat, T)
        step_ms = D.max_over_ranks(10.0 + rank)             # device time = max over ranks
        out[rank] = (lo, hi, w_hat.numpy(), gw.numpy(), gc.numpy().copy(), step_ms)
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world,n_seq", [(2, 6), (3, 7), (3, 2)])
def test_sharded_ranks_match_the_single_process_batch(world, n_seq):
    oracle.build()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, _free_port(), n_seq, out), nprocs=world, join=True)
        res = dict(out)
    c = I.codebook(1 << L, seed=11)
    w = I.weights(n_seq, SEQ_LEN, seed=12)
    g = I.upstream_grad(n_seq, SEQ_LEN, seed=13)
    what_all, _, _ = oracle.forward(w, c, T, L, K_BITS, nthreads=1)
    gw_all, gc_all = oracle.backward(g, w, c, T, L, K_BITS, nthreads=1)
    covered = sorted((res[r][0], res[r][1]) for r in range(world))
    assert covered[0][0] == 0 and covered[-1][1] == n_seq
    assert all(a[1] == b[0] for a, b in zip(covered, covered[1:]))
    for r in range(world):
        lo, hi, w_hat, gw, gc, step_ms = res[r]
        assert w_hat.shape == (hi - lo, SEQ_LEN)
        np.testing.assert_allclose(w_hat, what_all[lo:hi], rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(gw, gw_all[lo:hi], rtol=1e-12, atol=1e-14)
        # float32 sum of per-rank float32 partials against the float64 whole
        np.testing.assert_allclose(gc, gc_all, rtol=1e-5, atol=1e-6)
        assert step_ms == 10.0 + world - 1


@pytest.mark.parametrize("n_seq,world", [(0, 1), (1, 4), (7, 3), (65536, 8), (10, 10)])
def test_shard_bounds_partition_the_batch(n_seq, world):
    bounds = [D.shard_bounds(n_seq, world, r) for r in range(world)]
    assert bounds[0][0] == 0 and bounds[-1][1] == n_seq
    assert all(a[1] == b[0] for a, b in zip(bounds, bounds[1:]))
    sizes = [hi - lo for lo, hi in bounds]
    assert max(sizes) - min(sizes) <= 1 and sizes == sorted(sizes, reverse=True)


def test_shard_bounds_rejects_bad_ranks():
    with pytest.raises(ValueError):
        D.shard_bounds(4, 2, 2)
    with pytest.raises(ValueError):
        D.shard_bounds(4, 0, 0)
