"""Write the oracle's results on 256-sequence subsets of the two large
bitshift workloads (expected values for tests/test_gpu_subset_parity.py).

    python tests/golden/make_subset_parity.py [--threads N] [--only NAME]

The float64 oracle takes seconds per sequence at 2^16 states, so the
256-sequence subsets (about 40 minutes of CPU on 8 cores) are computed once
here instead of inside every GPU test run.  This script calls only the oracle
package and the seeded input generators; nothing in it comes from the CUDA
library.  The subsets are the first 256 rows of

  * the 2048 x 8192 projection (2^16 states, k = 2, 256 steps) at the first
    and the last temperature of its annealing sweep (0.3 and 0.005);
  * the bit-width sweep (2^16 states, 256 steps, T = 0.1) at k = 3 and k = 4.

Each file holds float32 copies of w_hat [256][256], grad_w [256][256],
grad_codebook [65536] (summed over the 256 sequences) and float64 log_z [256].
The upstream gradient is the workload's (seed 2); the backward call's soft
codeword input only centres the accumulators, so the oracle's own is used.
"""
from __future__ import annotations

import argparse
import os
import sys
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bcjr_inputs as I  # noqa: E402
import oracle  # noqa: E402

SUBSET = 256


def cases():
    proj = I.WORKLOADS["proj2048x8192_L16_k2"]
    bw = I.WORKLOADS["bitwidth_L16_k234"]
    temps = proj["T"]
    return {
        "proj_T0": dict(L=proj["state_bits"], k=proj["k"], n=proj["seq_len"], T=temps[0]),
        "proj_T7": dict(L=proj["state_bits"], k=proj["k"], n=proj["seq_len"], T=temps[-1]),
        "bitwidth_k3": dict(L=bw["state_bits"], k=3, n=bw["seq_len"], T=bw["T"][0]),
        "bitwidth_k4": dict(L=bw["state_bits"], k=4, n=bw["seq_len"], T=bw["T"][0]),
    }


def path(name: str) -> str:
    return os.path.join(HERE, f"subset_{name}.npz")


def inputs(L: int, n: int):
    """The first SUBSET rows of the workloads' weights and upstream gradient
    (the generators fill rows in order, so these are the full tensors' rows)."""
    return I.codebook(1 << L), I.weights(SUBSET, n), I.upstream_grad(SUBSET, n)


def make(name: str, threads: int):
    cfg = cases()[name]
    L, k, n, T = cfg["L"], cfg["k"], cfg["n"], cfg["T"]
    c, w, g = inputs(L, n)
    t0 = time.time()
    w_hat, log_z, _ = oracle.forward(w, c, T, L, k, nthreads=threads)
    grad_w, grad_c = oracle.backward(g, w, c, T, L, k, nthreads=threads)
    np.savez(path(name), w_hat=w_hat.astype(np.float32), log_z=log_z, grad_w=grad_w.astype(np.float32),
             grad_codebook=grad_c.astype(np.float32), L=L, k=k, n=n, T=T, n_seq=SUBSET)
    print(f"{name}: L={L} k={k} n={n} T={T:.6g} in {time.time() - t0:.0f} s -> {path(name)}", flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--threads", type=int, default=0)
    ap.add_argument("--only", default="")
    a = ap.parse_args()
    oracle.build()
    for name in cases():
        if a.only and name != a.only:
            continue
        make(name, a.threads)


if __name__ == "__main__":
    main()
