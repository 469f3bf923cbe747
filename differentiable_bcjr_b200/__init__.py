"""differentiable_bcjr_b200 -- B200 (sm_100a) kernels for the BCJR-QAT hot path.

A thin ctypes binding over libbcjr.so (C ABI in include/bcjr.h).  This module
only marshals arguments: PyTorch supplies device memory and the current CUDA
stream, every step of the computation runs in the library's kernels.  There
is no CPU fallback: if the library is missing or no CUDA device is present,
the calls raise.

  bcjr_forward(w, codebook, T, state_bits, k)        -> (w_hat, marginals|None, log_z)
  bcjr_backward(grad_w_hat, w, codebook, w_hat, T, state_bits, k) -> (grad_w, grad_codebook)
  viterbi_decode(w, codebook, state_bits, k)          -> (states, w_hard)
  bcjr_dense_forward / bcjr_dense_backward            (fully connected trellis)
  bcjr_dense_backward(..., want_grad_log_trans=True)  (also dL/dLambda, tensor cores)
  SoftTrellisQuant, DenseTrellisQuant                 torch.autograd.Function
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "LIB_PATH", "lib", "BCJRError", "bcjr_forward", "bcjr_backward", "viterbi_decode",
    "bcjr_dense_forward", "bcjr_dense_backward", "workspace_size", "Workspace",
    "SoftTrellisQuant", "soft_quantize", "DenseTrellisQuant", "dense_soft_quantize", "bcjr_forward_static_scratch",
    "static_scratch_status", "probe_xu", "probe_mma_tf32", "probe_dsmem", "OP_FORWARD", "OP_BACKWARD", "OP_VITERBI",
    "OP_DENSE_FORWARD", "OP_DENSE_BACKWARD", "OP_DENSE_BACKWARD_LAMBDA", "STATUS",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libbcjr.so")

OP_FORWARD, OP_BACKWARD, OP_VITERBI, OP_DENSE_FORWARD, OP_DENSE_BACKWARD, OP_DENSE_BACKWARD_LAMBDA = range(6)
STATUS = {0: "BCJR_OK", 1: "BCJR_ERR_INVALID_ARG", 2: "BCJR_ERR_UNSUPPORTED", 3: "BCJR_ERR_WORKSPACE",
          4: "BCJR_ERR_CUDA", 5: "BCJR_ERR_TIMEOUT", 6: "BCJR_ERR_NONFINITE"}


class BCJRError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {lib().bcjr_status_string(status).decode()}")


class Options(ctypes.Structure):
    _fields_ = [("checkpoint_interval", ctypes.c_int), ("sequences_in_flight", ctypes.c_int),
                ("timeout_probe_cycles", ctypes.c_int), ("reserved", ctypes.c_int * 5)]


_lib = None
_P = ctypes.c_void_p
_F = ctypes.c_float
_I = ctypes.c_int
_Z = ctypes.c_size_t

_SIGS = {
    "bcjr_workspace_size": (_Z, [_I, _I, _I, _I, _I, ctypes.POINTER(Options)]),
    "bcjr_forward": (_I, [_P, _P, _F, _I, _I, _I, _I, _P, _P, _P, ctypes.POINTER(Options), _P, _Z, _P]),
    "bcjr_forward_static_scratch": (_I, [_P, _P, _F, _I, _I, _I, _I, _P, _P, _P, ctypes.POINTER(Options), _P]),
    "bcjr_backward": (_I, [_P, _P, _P, _P, _F, _I, _I, _I, _I, _P, _P, _I, ctypes.POINTER(Options), _P, _Z,
                           _P]),
    "viterbi_decode": (_I, [_P, _P, _I, _I, _I, _I, _P, _P, _P, _Z, _P]),
    "bcjr_dense_forward": (_I, [_P, _P, _P, _F, _I, _I, _I, _P, _P, _P, ctypes.POINTER(Options), _P, _Z, _P]),
    "bcjr_dense_backward": (_I, [_P, _P, _P, _P, _P, _F, _I, _I, _I, _P, _P, _I, ctypes.POINTER(Options), _P,
                                 _Z, _P]),
    "bcjr_dense_backward_lambda": (_I, [_P, _P, _P, _P, _P, _F, _I, _I, _I, _P, _P, _P, _I,
                                        ctypes.POINTER(Options), _P, _Z, _P]),
    "bcjr_get_status": (_I, [_P, _P]),
    "bcjr_static_scratch_status": (_I, [_P]),
    "bcjr_status_string": (ctypes.c_char_p, [_I]),
    "bcjr_probe_xu": (_I, [_I, _I, _P, _P, _I, _P]),
    "bcjr_probe_mma_tf32": (_I, [_I, _I, _P, _P, _I, _P]),
    "bcjr_probe_dsmem": (_I, [_I, _I, _P, _P, _I, _P]),
    "bcjr_probe_dsmem_bulk": (_I, [_I, _I, _I, _P, _P, _I, _P]),
    "bcjr_version": (_I, []),
}


def lib():
    """The loaded libbcjr (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m differentiable_bcjr_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _opts(checkpoint_interval: int = 0, sequences_in_flight: int = 0, timeout_probe_cycles: int = 0):
    o = Options()
    o.checkpoint_interval = int(checkpoint_interval)
    o.sequences_in_flight = int(sequences_in_flight)
    o.timeout_probe_cycles = int(timeout_probe_cycles)
    return o


def _stream(device=None) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _need_cuda(*ts):
    for t in ts:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("libbcjr works on CUDA tensors only (no CPU path)")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")


def _expect(t, name, shape, dtype, device):
    if t is None:
        return
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, not {tuple(t.shape)}")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, not {t.dtype}")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, the weights on {device}")


def _weights_2d(w):
    if w.dim() != 2:
        raise ValueError("w must be [n_seq][seq_len]")
    if w.dtype != torch.float32:
        raise ValueError(f"w must be torch.float32, not {w.dtype}")
    return w.shape


def _ptr(t):
    return None if t is None else t.data_ptr()


def workspace_size(op: int, state_bits: int, k: int, seq_len: int, n_seq: int, checkpoint_interval: int = 0) -> int:
    o = _opts(checkpoint_interval)
    return int(lib().bcjr_workspace_size(op, state_bits, k, seq_len, n_seq, ctypes.byref(o)))


class Workspace:
    """A reusable device workspace that grows on demand (one per stream)."""

    def __init__(self, device=None):
        self.device = torch.device(device or "cuda")
        self.buf = None

    def get(self, nbytes: int) -> torch.Tensor:
        nbytes = max(int(nbytes), 256)
        if self.buf is None or self.buf.numel() < nbytes:
            self.buf = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
        return self.buf


_default_ws = {}


def _ws(device, nbytes, ws):
    if ws is None:
        key = (torch.device(device).index, torch.cuda.current_stream(device).cuda_stream)
        ws = _default_ws.setdefault(key, Workspace(device))
    return ws.get(nbytes)


def _check(status: int, what: str):
    if status != 0:
        raise BCJRError(status, what)


def get_status(ws_tensor: torch.Tensor) -> int:
    return int(lib().bcjr_get_status(ws_tensor.data_ptr(), _stream(ws_tensor.device)))


def bcjr_forward(w, codebook, T, state_bits, k, want_marginals=False, checkpoint_interval=0, ws=None,
                 out=None, sequences_in_flight=0, timeout_probe_cycles=0):
    """Soft codeword of every row of w [N][n] (float32, CUDA).  Returns
    (w_hat [N][n], marginals [N][n][S] or None, log_z [N]).
    `timeout_probe_cycles` is the testing aid of bcjr_options (see bcjr.h)."""
    _need_cuda(w, codebook, out)
    N, n = _weights_2d(w)
    S = 1 << state_bits
    dev = w.device
    _expect(codebook, "codebook", (S,), torch.float32, dev)
    _expect(out, "out", (N, n), torch.float32, dev)
    w_hat = out if out is not None else torch.empty((N, n), dtype=torch.float32, device=dev)
    marg = torch.empty((N, n, S), dtype=torch.float32, device=dev) if want_marginals else None
    log_z = torch.empty((N,), dtype=torch.float32, device=dev)
    o = _opts(checkpoint_interval, sequences_in_flight, timeout_probe_cycles)
    nbytes = lib().bcjr_workspace_size(OP_FORWARD, state_bits, k, n, N, ctypes.byref(o))
    if nbytes == 0:
        raise BCJRError(2, "bcjr_workspace_size")
    wsb = _ws(dev, nbytes, ws)
    _check(lib().bcjr_forward(_ptr(w), _ptr(codebook), float(T), state_bits, k, n, N, _ptr(w_hat), _ptr(marg),
                              _ptr(log_z), ctypes.byref(o), _ptr(wsb), wsb.numel(), _stream(dev)),
           "bcjr_forward")
    return w_hat, marg, log_z


STATIC_SCRATCH_BYTES = 32 << 20


def bcjr_forward_static_scratch(w, codebook, T, state_bits, k, w_hat, log_z=None, marginals=None,
                                checkpoint_interval=0):
    """bcjr_forward into caller-provided outputs, with the library's static
    device scratch as workspace: neither this function nor the library
    allocates device memory.  Calls on one device share that scratch, so they
    must not overlap in time.  Every tensor must sit on w's device, which is
    made current for the call."""
    _need_cuda(w, codebook, w_hat, log_z, marginals)
    if w.dim() != 2:
        raise ValueError("w must be [n_seq][seq_len]")
    N, n = w.shape
    S = 1 << int(state_bits)
    dev = w.device
    _expect(w, "w", (N, n), torch.float32, dev)
    _expect(codebook, "codebook", (S,), torch.float32, dev)
    _expect(w_hat, "w_hat", (N, n), torch.float32, dev)
    _expect(log_z, "log_z", (N,), torch.float32, dev)
    _expect(marginals, "marginals", (N, n, S), torch.float32, dev)
    o = _opts(checkpoint_interval)
    with torch.cuda.device(dev):
        _check(lib().bcjr_forward_static_scratch(_ptr(w), _ptr(codebook), float(T), state_bits, k, n, N,
                                                 _ptr(w_hat), _ptr(marginals), _ptr(log_z), ctypes.byref(o),
                                                 _stream(dev)), "bcjr_forward_static_scratch")


def static_scratch_status(device=None) -> int:
    """Synchronise the current stream of `device` and return the device-side
    status (a bcjr_status code) of the last bcjr_forward_static_scratch call
    on that device."""
    dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    with torch.cuda.device(dev):
        return int(lib().bcjr_static_scratch_status(_stream(dev)))


def bcjr_backward(grad_w_hat, w, codebook, w_hat, T, state_bits, k, checkpoint_interval=0, ws=None,
                  grad_codebook=None, accumulate_codebook=False, sequences_in_flight=0, grad_w_out=None):
    """VJP of the soft codeword.  Returns (grad_w [N][n], grad_codebook [S]); grad_w goes
    into `grad_w_out` when given."""
    _need_cuda(grad_w_hat, w, codebook, w_hat, grad_w_out, grad_codebook)
    N, n = _weights_2d(w)
    S = 1 << state_bits
    for t, name, shape in ((grad_w_hat, "grad_w_hat", (N, n)), (w_hat, "w_hat", (N, n)),
                           (grad_w_out, "grad_w_out", (N, n)), (codebook, "codebook", (S,)),
                           (grad_codebook, "grad_codebook", (S,))):
        _expect(t, name, shape, torch.float32, w.device)
    dev = w.device
    grad_w = grad_w_out if grad_w_out is not None else torch.empty((N, n), dtype=torch.float32, device=dev)
    if grad_codebook is None:
        grad_codebook = torch.empty((S,), dtype=torch.float32, device=dev)
        accumulate_codebook = False
    o = _opts(checkpoint_interval, sequences_in_flight)
    nbytes = lib().bcjr_workspace_size(OP_BACKWARD, state_bits, k, n, N, ctypes.byref(o))
    if nbytes == 0:
        raise BCJRError(2, "bcjr_workspace_size")
    wsb = _ws(dev, nbytes, ws)
    _check(lib().bcjr_backward(_ptr(grad_w_hat), _ptr(w), _ptr(codebook), _ptr(w_hat), float(T), state_bits, k,
                               n, N, _ptr(grad_w), _ptr(grad_codebook), int(bool(accumulate_codebook)),
                               ctypes.byref(o), _ptr(wsb), wsb.numel(), _stream(dev)), "bcjr_backward")
    return grad_w, grad_codebook


def viterbi_decode(w, codebook, state_bits, k, ws=None):
    """Hard (T -> 0) decode.  Returns (states int32 [N][n], w_hard [N][n])."""
    _need_cuda(w, codebook)
    N, n = _weights_2d(w)
    _expect(codebook, "codebook", (1 << state_bits,), torch.float32, w.device)
    dev = w.device
    states = torch.empty((N, n), dtype=torch.int32, device=dev)
    w_hard = torch.empty((N, n), dtype=torch.float32, device=dev)
    nbytes = lib().bcjr_workspace_size(OP_VITERBI, state_bits, k, n, N, None)
    if nbytes == 0:
        raise BCJRError(2, "bcjr_workspace_size")
    wsb = _ws(dev, nbytes, ws)
    _check(lib().viterbi_decode(_ptr(w), _ptr(codebook), state_bits, k, n, N, _ptr(states), _ptr(w_hard),
                                _ptr(wsb), wsb.numel(), _stream(dev)), "viterbi_decode")
    return states, w_hard


def _log2_states(S: int) -> int:
    b = S.bit_length() - 1
    if 1 << b != S:
        raise ValueError("n_states must be a power of two")
    return b


def bcjr_dense_forward(w, codebook, log_trans, T, want_marginals=False, checkpoint_interval=0, ws=None):
    _need_cuda(w, codebook, log_trans)
    N, n = _weights_2d(w)
    S = codebook.shape[0]
    _expect(codebook, "codebook", (S,), torch.float32, w.device)
    _expect(log_trans, "log_trans", (S, S), torch.float32, w.device)
    dev = w.device
    w_hat = torch.empty((N, n), dtype=torch.float32, device=dev)
    marg = torch.empty((N, n, S), dtype=torch.float32, device=dev) if want_marginals else None
    log_z = torch.empty((N,), dtype=torch.float32, device=dev)
    o = _opts(checkpoint_interval)
    nbytes = lib().bcjr_workspace_size(OP_DENSE_FORWARD, _log2_states(S), 0, n, N, ctypes.byref(o))
    if nbytes == 0:
        raise BCJRError(2, "bcjr_workspace_size")
    wsb = _ws(dev, nbytes, ws)
    _check(lib().bcjr_dense_forward(_ptr(w), _ptr(codebook), _ptr(log_trans), float(T), S, n, N, _ptr(w_hat),
                                    _ptr(marg), _ptr(log_z), ctypes.byref(o), _ptr(wsb), wsb.numel(),
                                    _stream(dev)), "bcjr_dense_forward")
    return w_hat, marg, log_z


def bcjr_dense_backward(grad_w_hat, w, codebook, log_trans, w_hat, T, checkpoint_interval=0, ws=None,
                        want_grad_log_trans=False, grad_codebook=None, grad_log_trans=None, accumulate=False):
    """VJP of the dense soft codeword: (grad_w [N][n], grad_codebook [S]) and,
    with want_grad_log_trans, grad_log_trans [S][S] as a third result.  Given
    `grad_codebook` / `grad_log_trans` tensors, the results go there, added to
    their contents when `accumulate` is set."""
    _need_cuda(grad_w_hat, w, codebook, log_trans, w_hat, grad_codebook, grad_log_trans)
    N, n = _weights_2d(w)
    S = codebook.shape[0]
    for t, name, shape in ((grad_w_hat, "grad_w_hat", (N, n)), (w_hat, "w_hat", (N, n)), (codebook, "codebook", (S,)),
                           (log_trans, "log_trans", (S, S)), (grad_codebook, "grad_codebook", (S,)),
                           (grad_log_trans, "grad_log_trans", (S, S))):
        _expect(t, name, shape, torch.float32, w.device)
    dev = w.device
    grad_w = torch.empty((N, n), dtype=torch.float32, device=dev)
    if grad_codebook is None or (want_grad_log_trans and grad_log_trans is None):
        accumulate = False
    grad_c = grad_codebook if grad_codebook is not None else torch.empty((S,), dtype=torch.float32, device=dev)
    o = _opts(checkpoint_interval)
    op = OP_DENSE_BACKWARD_LAMBDA if want_grad_log_trans else OP_DENSE_BACKWARD
    nbytes = lib().bcjr_workspace_size(op, _log2_states(S), 0, n, N, ctypes.byref(o))
    if nbytes == 0:
        raise BCJRError(2, "bcjr_workspace_size")
    wsb = _ws(dev, nbytes, ws)
    if not want_grad_log_trans:
        _check(lib().bcjr_dense_backward(_ptr(grad_w_hat), _ptr(w), _ptr(codebook), _ptr(log_trans), _ptr(w_hat),
                                         float(T), S, n, N, _ptr(grad_w), _ptr(grad_c), int(bool(accumulate)),
                                         ctypes.byref(o), _ptr(wsb), wsb.numel(), _stream(dev)),
               "bcjr_dense_backward")
        return grad_w, grad_c
    grad_lam = grad_log_trans if grad_log_trans is not None else torch.empty((S, S), dtype=torch.float32,
                                                                             device=dev)
    _check(lib().bcjr_dense_backward_lambda(_ptr(grad_w_hat), _ptr(w), _ptr(codebook), _ptr(log_trans),
                                            _ptr(w_hat), float(T), S, n, N, _ptr(grad_w), _ptr(grad_c),
                                            _ptr(grad_lam), int(bool(accumulate)), ctypes.byref(o), _ptr(wsb),
                                            wsb.numel(), _stream(dev)), "bcjr_dense_backward_lambda")
    return grad_w, grad_c, grad_lam


class SoftTrellisQuant(torch.autograd.Function):
    """w_hat = BCJR soft codeword of w at temperature T (differentiable in w and codebook)."""

    @staticmethod
    def forward(ctx, w, codebook, T, state_bits, k):
        w_c = w.contiguous()
        c_c = codebook.contiguous()
        w_hat, _, _ = bcjr_forward(w_c, c_c, T, state_bits, k)
        ctx.save_for_backward(w_c, c_c, w_hat)
        ctx.cfg = (float(T), int(state_bits), int(k))
        return w_hat

    @staticmethod
    def backward(ctx, grad_w_hat):
        w, c, w_hat = ctx.saved_tensors
        T, L, k = ctx.cfg
        gw, gc = bcjr_backward(grad_w_hat.contiguous().float(), w, c, w_hat, T, L, k)
        return gw, gc, None, None, None


def soft_quantize(w, codebook, T, state_bits, k):
    return SoftTrellisQuant.apply(w, codebook, T, state_bits, k)


class DenseTrellisQuant(torch.autograd.Function):
    """w_hat = soft codeword of w over the dense 256-state trellis with
    log-transitions `log_trans` (differentiable in w, codebook and log_trans;
    the log_trans gradient is computed only when it is required)."""

    @staticmethod
    def forward(ctx, w, codebook, log_trans, T):
        w_c, c_c, l_c = w.contiguous(), codebook.contiguous(), log_trans.contiguous()
        w_hat, _, _ = bcjr_dense_forward(w_c, c_c, l_c, T)
        ctx.save_for_backward(w_c, c_c, l_c, w_hat)
        ctx.T = float(T)
        return w_hat

    @staticmethod
    def backward(ctx, grad_w_hat):
        w, c, lam, w_hat = ctx.saved_tensors
        g = grad_w_hat.contiguous().float()
        if ctx.needs_input_grad[2]:
            gw, gc, gl = bcjr_dense_backward(g, w, c, lam, w_hat, ctx.T, want_grad_log_trans=True)
        else:
            (gw, gc), gl = bcjr_dense_backward(g, w, c, lam, w_hat, ctx.T), None
        return gw, gc, gl, None


def dense_soft_quantize(w, codebook, log_trans, T):
    return DenseTrellisQuant.apply(w, codebook, log_trans, T)


def probe_xu(op: str = "ex2", iters: int = 4096, device=None) -> dict:
    """Measured throughput of the special-function pipe (bcjr_probe.h): ex2
    or lg2 instructions per clock per SM, from each CTA's own cycle count
    (one CTA per SM).  Returns {"ops_per_clk_per_sm": median over SMs, "min",
    "max", "sms", "ops"}."""
    dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    code = {"ex2": 0, "lg2": 1}[op]
    sink = torch.empty(sms * 1024, dtype=torch.float32, device=dev)
    cycles = torch.zeros(sms, dtype=torch.int64, device=dev)
    with torch.cuda.device(dev):
        _check(lib().bcjr_probe_xu(code, int(iters), _ptr(sink), _ptr(cycles), sms, _stream(dev)), "bcjr_probe_xu")
        torch.cuda.synchronize(dev)
    ops = 1024 * 16 * int(iters)
    rates = sorted(ops / float(c) for c in cycles.cpu().tolist())
    return {"ops_per_clk_per_sm": rates[len(rates) // 2], "min": rates[0], "max": rates[-1], "sms": sms,
            "ops": ops * sms}


def probe_mma_tf32(n: int = 64, iters: int = 4096, device=None) -> dict:
    """Issue cost of one tcgen05 tf32 product with operand A in tensor memory
    (bcjr_probe.h), M = 128, K = 8 and the given N, one CTA per SM.  Returns
    {"clk_per_mma", "mac_per_clk_per_sm"} (medians over SMs), "sms"."""
    dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    cycles = torch.zeros(sms, dtype=torch.int64, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    with torch.cuda.device(dev):
        _check(lib().bcjr_probe_mma_tf32(int(n), int(iters), _ptr(cycles), _ptr(status), sms, _stream(dev)),
               "bcjr_probe_mma_tf32")
        torch.cuda.synchronize(dev)
    if int(status.item()) != 0:
        raise BCJRError(int(status.item()), "bcjr_probe_mma_tf32: a wait ran out")
    c = sorted(float(v) for v in cycles.cpu().tolist())
    med = c[len(c) // 2]
    return {"clk_per_mma": med / iters, "mac_per_clk_per_sm": 128.0 * n * 8 * iters / med, "sms": sms}


def probe_dsmem(reps: int = 4, rounds: int = 100, clusters: int = 0, device=None, chunk: int = 0) -> dict:
    """Bandwidth of the exchange between the CTAs of 4-CTA clusters
    (bcjr_probe.h): per-thread st.async stores (chunk = 0) or bulk copies of
    `chunk` bytes (bcjr_probe_dsmem_bulk).  clusters = 0: one per 4 SMs.
    Returns {"bytes_per_clk_per_sm": median over CTAs of the bytes each sends
    per clock, "min", "max", "ctas"}."""
    dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    ncl = int(clusters) if clusters > 0 else sms // 4
    cycles = torch.zeros(4 * ncl, dtype=torch.int64, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    name = "bcjr_probe_dsmem_bulk" if chunk else "bcjr_probe_dsmem"
    with torch.cuda.device(dev):
        if chunk:
            rc = lib().bcjr_probe_dsmem_bulk(int(chunk), int(reps), int(rounds), _ptr(cycles), _ptr(status), ncl,
                                             _stream(dev))
        else:
            rc = lib().bcjr_probe_dsmem(int(reps), int(rounds), _ptr(cycles), _ptr(status), ncl, _stream(dev))
        _check(rc, name)
        torch.cuda.synchronize(dev)
    if int(status.item()) != 0:
        raise BCJRError(int(status.item()), name + ": a wait ran out")
    out = 3 * 32768 * int(reps) * int(rounds)
    r = sorted(out / float(v) for v in cycles.cpu().tolist())
    return {"bytes_per_clk_per_sm": r[len(r) // 2], "min": r[0], "max": r[-1], "ctas": 4 * ncl}

