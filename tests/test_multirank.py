"""Multi-rank host logic on CPU (two `gloo` ranks, no GPU).

The path shards by sequence: every rank owns whole sequences, and the one
cross-rank exchange is the all-reduce (sum) of grad_codebook.  Here each rank
computes its shard with the oracle and the all-reduced codebook gradient must
equal the single-process gradient of the concatenated batch; the step time is
reduced with MAX, as the benchmark does.
"""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bcjr_inputs as I
import oracle

L, K_BITS, N_SEQ, SEQ_LEN, T = 6, 2, 6, 5, 0.4


def _shard(rank, world, n_seq):
    per = (n_seq + world - 1) // world
    lo = min(n_seq, rank * per)
    return lo, min(n_seq, lo + per)


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        c = I.codebook(1 << L, seed=11)
        w = I.weights(N_SEQ, SEQ_LEN, seed=12)
        g = I.upstream_grad(N_SEQ, SEQ_LEN, seed=13)
        lo, hi = _shard(rank, world, N_SEQ)
        gw, gc = oracle.backward(g[lo:hi], w[lo:hi], c, T, L, K_BITS, nthreads=1)
        gct = torch.from_numpy(np.ascontiguousarray(gc))
        dist.all_reduce(gct)                                   # the path's only exchange
        step_ms = torch.tensor([10.0 + rank], dtype=torch.float64)
        dist.all_reduce(step_ms, op=dist.ReduceOp.MAX)         # device time = max over ranks
        out[rank] = (lo, hi, gw, gct.numpy(), float(step_ms.item()))
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_ranks_shard_sequences_and_sum_the_codebook_gradient():
    oracle.build()
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    c = I.codebook(1 << L, seed=11)
    w = I.weights(N_SEQ, SEQ_LEN, seed=12)
    g = I.upstream_grad(N_SEQ, SEQ_LEN, seed=13)
    gw_all, gc_all = oracle.backward(g, w, c, T, L, K_BITS, nthreads=1)
    covered = sorted((res[r][0], res[r][1]) for r in range(world))
    assert covered[0][0] == 0 and covered[-1][1] == N_SEQ
    assert all(a[1] == b[0] for a, b in zip(covered, covered[1:]))
    for r in range(world):
        lo, hi, gw, gc, step_ms = res[r]
        np.testing.assert_allclose(gw, gw_all[lo:hi], rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(gc, gc_all, rtol=1e-12, atol=1e-12)
        assert step_ms == 10.0 + world - 1
