"""Brute-force enumeration of every trellis path (test infrastructure only).

Independent of the recursions in bcjr_oracle.c: it lists all state paths the
trellis allows, weights each path by exp(sum_t phi_t(s_t)) (plus the dense
log-transitions), and reads the quantities the paper defines straight off the
path distribution ("BCJR-QAT", technical summary, "core mechanism": marginal
posteriors of the states under the Boltzmann distribution over paths, and the
soft codeword as the Boltzmann expectation of the emitted codeword):

  gamma_t(s) = P(s_t = s)         w_hat_t = E[c(s_t)]         log Z

and the vector-Jacobian product of L = sum_t g_t w_hat_t from the covariance
identity d E_p[f] / d theta = E[df/dtheta] + Cov(f, dE/dtheta) (E the path
log-weight), with no forward or backward recursion anywhere:

  dL/dw_u  = (2/T) Cov(G, c(s_u))
  dL/dc(r) = sum_u g_u P(s_u = r) + (2/T) sum_u (w_u - c(r)) Cov(G, 1[s_u = r])
  dL/dLam[p][r] = Cov(G, number of transitions p -> r on the path)      (dense)

where G = sum_t g_t c(s_t).  Also the minimum-distortion (T -> 0) path.
Sizes: S * 2^(k (n-1)) bitshift paths, S^n dense paths; keep them below ~1e6.
"""
from __future__ import annotations

import numpy as np


def bitshift_paths(state_bits: int, k: int, seq_len: int) -> np.ndarray:
    """Every state path allowed by the bitshift trellis: int64 [P][n]."""
    S, K = 1 << state_bits, 1 << k
    paths = np.arange(S, dtype=np.int64)[:, None]
    for _ in range(1, seq_len):
        last = paths[:, -1]
        nxt = ((last[:, None] << k) & (S - 1)) | np.arange(K, dtype=np.int64)[None, :]
        paths = np.concatenate([np.repeat(paths, K, axis=0), nxt.reshape(-1, 1)], axis=1)
    return paths


def dense_paths(n_states: int, seq_len: int) -> np.ndarray:
    """Every path of a fully connected trellis: int64 [S^n][n]."""
    grids = np.meshgrid(*[np.arange(n_states, dtype=np.int64)] * seq_len, indexing="ij")
    return np.stack([g.reshape(-1) for g in grids], axis=1)


def _as64(x) -> np.ndarray:
    a = x.detach().cpu().numpy() if hasattr(x, "detach") else np.asarray(x)
    return np.asarray(a, dtype=np.float32).astype(np.float64)


def _path_stats(paths, w_row, c, T, g_row=None, log_trans=None):
    n = paths.shape[1]
    S = c.shape[0]
    cw = c[paths]                                   # [P][n] codeword emitted at each step
    energy = -((w_row[None, :] - cw) ** 2).sum(axis=1) / T
    if log_trans is not None:
        energy = energy + log_trans[paths[:, :-1], paths[:, 1:]].sum(axis=1)
    m = energy.max()
    p = np.exp(energy - m)
    z = p.sum()
    p /= z
    log_z = m + np.log(z)
    gamma = np.zeros((n, S))
    for t in range(n):
        np.add.at(gamma[t], paths[:, t], p)
    w_hat = (p[:, None] * cw).sum(axis=0)
    out = dict(log_z=log_z, gamma=gamma, w_hat=w_hat)
    if g_row is not None:
        G = (g_row[None, :] * cw).sum(axis=1)
        Gc = G - (p * G).sum()
        grad_w = (2.0 / T) * (p[:, None] * Gc[:, None] * (cw - w_hat[None, :])).sum(axis=0)
        cov_ind = np.zeros((n, S))                  # Cov(G, 1[s_u = r])
        for t in range(n):
            np.add.at(cov_ind[t], paths[:, t], p * Gc)
        grad_c = (g_row[:, None] * gamma).sum(axis=0) + (2.0 / T) * (
            (w_row[:, None] - c[None, :]) * cov_ind).sum(axis=0)
        out.update(grad_w=grad_w, grad_c=grad_c)
        if log_trans is not None:
            cov_tr = np.zeros((S, S))               # Cov(G, #transitions p -> r)
            for t in range(1, n):
                np.add.at(cov_tr, (paths[:, t - 1], paths[:, t]), p * Gc)
            out.update(grad_lam=cov_tr)
    return out


def forward(w, codebook, T, state_bits, k):
    """(w_hat [N][n], log_z [N], gamma [N][n][S]) by path enumeration."""
    w = _as64(w)
    c = _as64(codebook)
    paths = bitshift_paths(state_bits, k, w.shape[1])
    res = [_path_stats(paths, w[i], c, float(T)) for i in range(w.shape[0])]
    return (np.stack([r["w_hat"] for r in res]), np.array([r["log_z"] for r in res]),
            np.stack([r["gamma"] for r in res]))


def backward(grad_w_hat, w, codebook, T, state_bits, k):
    """(grad_w [N][n], grad_codebook [S]) from the covariance identity."""
    w = _as64(w)
    g = _as64(grad_w_hat)
    c = _as64(codebook)
    paths = bitshift_paths(state_bits, k, w.shape[1])
    res = [_path_stats(paths, w[i], c, float(T), g_row=g[i]) for i in range(w.shape[0])]
    return np.stack([r["grad_w"] for r in res]), np.sum([r["grad_c"] for r in res], axis=0)


def min_distortion_paths(w, codebook, state_bits, k):
    """(paths [N][n], distortion [N], gap [N]): the least sum_t (w_t - c(s_t))^2
    path of each sequence, its distortion, and the gap to the second best path."""
    w = _as64(w)
    c = _as64(codebook)
    paths = bitshift_paths(state_bits, k, w.shape[1])
    out_p, out_d, out_gap = [], [], []
    for i in range(w.shape[0]):
        dist = ((w[i][None, :] - c[paths]) ** 2).sum(axis=1)
        order = np.argsort(dist, kind="stable")
        out_p.append(paths[order[0]])
        out_d.append(dist[order[0]])
        out_gap.append(dist[order[1]] - dist[order[0]] if len(order) > 1 else np.inf)
    return np.stack(out_p), np.array(out_d), np.array(out_gap)


def dense_forward(w, codebook, log_trans, T):
    w = _as64(w)
    c = _as64(codebook)
    lam = _as64(log_trans)
    paths = dense_paths(c.shape[0], w.shape[1])
    res = [_path_stats(paths, w[i], c, float(T), log_trans=lam) for i in range(w.shape[0])]
    return (np.stack([r["w_hat"] for r in res]), np.array([r["log_z"] for r in res]),
            np.stack([r["gamma"] for r in res]))


def dense_backward(grad_w_hat, w, codebook, log_trans, T):
    w = _as64(w)
    g = _as64(grad_w_hat)
    c = _as64(codebook)
    lam = _as64(log_trans)
    paths = dense_paths(c.shape[0], w.shape[1])
    res = [_path_stats(paths, w[i], c, float(T), g_row=g[i], log_trans=lam) for i in range(w.shape[0])]
    return (np.stack([r["grad_w"] for r in res]), np.sum([r["grad_c"] for r in res], axis=0),
            np.sum([r["grad_lam"] for r in res], axis=0))
