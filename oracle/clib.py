"""ctypes binding of the float64 C oracle (test infrastructure only).

Inputs are the exact float32 tensors handed to the GPU; the C code upcasts
them to float64.  Outputs are float64 numpy arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bcjr_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

_F = ctypes.POINTER(ctypes.c_float)
_D = ctypes.POINTER(ctypes.c_double)
_I = ctypes.POINTER(ctypes.c_int32)


def build(force: bool = False) -> str:
    """Compile bcjr_oracle.c into liboracle.so next to it."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fPIC", "-shared",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        for name in ("oracle_forward", "oracle_backward", "oracle_viterbi", "oracle_alpha_beta",
                     "oracle_dense_forward", "oracle_dense_backward", "oracle_max_threads"):
            getattr(lib, name).restype = ctypes.c_int
        _lib = lib
    return _lib


def _f32(x) -> np.ndarray:
    a = x.detach().cpu().numpy() if hasattr(x, "detach") else np.asarray(x)
    return np.ascontiguousarray(a, dtype=np.float32)


def _p(a: np.ndarray, t):
    return a.ctypes.data_as(t)


def _check(status: int, what: str):
    if status != 0:
        raise RuntimeError(f"{what}: oracle status {status}")


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def forward(w, codebook, T, state_bits, k, want_gamma=False, nthreads=0):
    """Soft codeword.  Returns (w_hat [N][n], log_z [N], gamma [N][n][S] or None)."""
    w = _f32(w)
    c = _f32(codebook)
    N, n = w.shape
    S = 1 << state_bits
    assert c.shape == (S,)
    w_hat = np.zeros((N, n))
    log_z = np.zeros(N)
    gamma = np.zeros((N, n, S)) if want_gamma else None
    _check(_load().oracle_forward(_p(w, _F), _p(c, _F), ctypes.c_double(float(T)), state_bits, k,
                                  n, N, _p(w_hat, _D),
                                  _p(gamma, _D) if gamma is not None else None,
                                  _p(log_z, _D), int(nthreads)), "oracle_forward")
    return w_hat, log_z, gamma


def backward(grad_w_hat, w, codebook, T, state_bits, k, nthreads=0):
    """VJP.  Returns (grad_w [N][n], grad_codebook [S] summed over sequences)."""
    g = _f32(grad_w_hat)
    w = _f32(w)
    c = _f32(codebook)
    N, n = w.shape
    S = 1 << state_bits
    assert g.shape == w.shape and c.shape == (S,)
    grad_w = np.zeros((N, n))
    grad_c = np.zeros(S)
    _check(_load().oracle_backward(_p(g, _F), _p(w, _F), _p(c, _F), ctypes.c_double(float(T)),
                                   state_bits, k, n, N, _p(grad_w, _D), _p(grad_c, _D),
                                   int(nthreads)), "oracle_backward")
    return grad_w, grad_c


def viterbi(w, codebook, state_bits, k, nthreads=0):
    """Max-sum hard decode.  Returns (states int32 [N][n], w_hard float32 [N][n], metric [N])."""
    w = _f32(w)
    c = _f32(codebook)
    N, n = w.shape
    states = np.zeros((N, n), dtype=np.int32)
    w_hard = np.zeros((N, n), dtype=np.float32)
    metric = np.zeros(N)
    _check(_load().oracle_viterbi(_p(w, _F), _p(c, _F), state_bits, k, n, N, _p(states, _I),
                                  _p(w_hard, _F), _p(metric, _D), int(nthreads)), "oracle_viterbi")
    return states, w_hard, metric


def alpha_beta(w_row, codebook, T, state_bits, k):
    """Full alpha and beta [n][S] (natural log) of one sequence."""
    w = _f32(w_row).reshape(-1)
    c = _f32(codebook)
    n = w.shape[0]
    S = 1 << state_bits
    alpha = np.zeros((n, S))
    beta = np.zeros((n, S))
    _check(_load().oracle_alpha_beta(_p(w, _F), _p(c, _F), ctypes.c_double(float(T)), state_bits, k,
                                     n, _p(alpha, _D), _p(beta, _D)), "oracle_alpha_beta")
    return alpha, beta


def dense_forward(w, codebook, log_trans, T, want_gamma=False, nthreads=0):
    w = _f32(w)
    c = _f32(codebook)
    lam = _f32(log_trans)
    N, n = w.shape
    S = c.shape[0]
    assert lam.shape == (S, S)
    w_hat = np.zeros((N, n))
    log_z = np.zeros(N)
    gamma = np.zeros((N, n, S)) if want_gamma else None
    _check(_load().oracle_dense_forward(_p(w, _F), _p(c, _F), _p(lam, _F), ctypes.c_double(float(T)),
                                        S, n, N, _p(w_hat, _D),
                                        _p(gamma, _D) if gamma is not None else None,
                                        _p(log_z, _D), int(nthreads)), "oracle_dense_forward")
    return w_hat, log_z, gamma


def dense_backward(grad_w_hat, w, codebook, log_trans, T, nthreads=0, want_grad_lam=False):
    """(grad_w [N][n], grad_c [S]) and, with want_grad_lam, grad_log_trans [S][S]."""
    g = _f32(grad_w_hat)
    w = _f32(w)
    c = _f32(codebook)
    lam = _f32(log_trans)
    N, n = w.shape
    S = c.shape[0]
    grad_w = np.zeros((N, n))
    grad_c = np.zeros(S)
    grad_lam = np.zeros((S, S)) if want_grad_lam else None
    _check(_load().oracle_dense_backward(_p(g, _F), _p(w, _F), _p(c, _F), _p(lam, _F),
                                         ctypes.c_double(float(T)), S, n, N, _p(grad_w, _D),
                                         _p(grad_c, _D), _p(grad_lam, _D) if grad_lam is not None else None,
                                         int(nthreads)), "oracle_dense_backward")
    return (grad_w, grad_c, grad_lam) if want_grad_lam else (grad_w, grad_c)
