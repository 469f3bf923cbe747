"""The C ABI library loads, exports what include/bcjr.h declares, and rejects
bad arguments on the host before touching the GPU (CPU only)."""
import ctypes
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bcjr.h")
HEADERS = sorted(glob.glob(os.path.join(ROOT, "include", "*.h")))


@pytest.fixture(scope="module")
def lib():
    from differentiable_bcjr_b200 import build
    path = build.build()
    return ctypes.CDLL(path)


def declared_functions():
    text = "\n".join(open(h).read() for h in HEADERS)
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*([a-z_][a-z0-9_]*)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_calls():
    names = declared_functions()
    for required in ["bcjr_forward", "bcjr_backward", "viterbi_decode", "bcjr_workspace_size",
                     "bcjr_get_status", "bcjr_status_string", "bcjr_dense_forward", "bcjr_dense_backward",
                     "bcjr_dense_backward_lambda", "bcjr_forward_static_scratch", "bcjr_static_scratch_status",
                     "bcjr_probe_xu", "bcjr_probe_mma_tf32", "bcjr_probe_dsmem",
                     "bcjr_probe_dsmem_bulk"]:
        assert required in names, names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    lib.bcjr_status_string.restype = ctypes.c_char_p
    for code in range(7):
        s = lib.bcjr_status_string(code).decode()
        assert s.startswith("BCJR_")
    assert lib.bcjr_version() >= 100


def _fwd(lib, w=1, c=1, T=0.5, L=8, k=2, n=4, N=2, what=1, ws=256, wsb=1 << 20):
    f = lib.bcjr_forward
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_float, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                  ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                  ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
    # fake, never-dereferenced addresses: validation must reject before any CUDA call
    P = lambda v: None if v == 0 else v * 4096
    return f(P(w), P(c), T, L, k, n, N, P(what), None, None, None, P(ws), wsb, None)


def test_invalid_arguments_are_rejected_on_the_host(lib):
    INVALID, UNSUPPORTED, WORKSPACE = 1, 2, 3
    assert _fwd(lib, w=0) == INVALID
    assert _fwd(lib, c=0) == INVALID
    assert _fwd(lib, what=0) == INVALID
    assert _fwd(lib, T=0.0) == INVALID
    assert _fwd(lib, T=-1.0) == INVALID
    assert _fwd(lib, T=float("inf")) == INVALID
    assert _fwd(lib, T=float("nan")) == INVALID
    assert _fwd(lib, n=0) == INVALID
    assert _fwd(lib, N=-1) == INVALID
    assert _fwd(lib, k=0) == INVALID
    assert _fwd(lib, k=9, L=8) == INVALID
    assert _fwd(lib, L=17, k=2) == UNSUPPORTED
    assert _fwd(lib, L=8, k=5) == UNSUPPORTED
    assert _fwd(lib, L=6, k=4) == UNSUPPORTED   # needs 2k <= state_bits
    assert _fwd(lib, ws=0) == WORKSPACE
    # misaligned workspace (not a multiple of 256 bytes)
    f = lib.bcjr_forward
    assert f(4096, 8192, 0.5, 8, 2, 4, 2, 12288, None, None, None, 4096 + 64, 1 << 20, None) == WORKSPACE


def test_viterbi_and_backward_reject_null_pointers(lib):
    v = lib.viterbi_decode
    v.restype = ctypes.c_int
    v.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                  ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
    assert v(None, 4096, 8, 2, 4, 2, 8192, None, 12288, 1 << 20, None) == 1
    assert v(4096, 4096, 8, 2, 4, 2, None, None, 12288, 1 << 20, None) == 1
    b = lib.bcjr_backward
    b.restype = ctypes.c_int
    b.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_float] + [ctypes.c_int] * 4 + [ctypes.c_void_p] * 2 + \
        [ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
    assert b(None, 4096, 4096, 4096, 0.5, 8, 2, 4, 2, 4096, 4096, 0, None, 4096, 1 << 20, None) == 1
    assert b(4096, 4096, 4096, None, 0.5, 8, 2, 4, 2, 4096, 4096, 0, None, 4096, 1 << 20, None) == 1


def test_get_status_rejects_null(lib):
    lib.bcjr_get_status.restype = ctypes.c_int
    lib.bcjr_get_status.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
    assert lib.bcjr_get_status(None, None) == 1


class _Opts(ctypes.Structure):
    _fields_ = [("checkpoint_interval", ctypes.c_int), ("sequences_in_flight", ctypes.c_int),
                ("reserved", ctypes.c_int * 6)]


class _BitshiftOpts(ctypes.Structure):
    _fields_ = [("checkpoint_interval", ctypes.c_int), ("sequences_in_flight", ctypes.c_int),
                ("timeout_probe_cycles", ctypes.c_int), ("reserved", ctypes.c_int * 5)]


def test_bitshift_options_are_checked_on_the_host(lib):
    INVALID = 1
    f = lib.bcjr_forward
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_float, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                  ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.POINTER(_BitshiftOpts),
                  ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
    for field, value in [("sequences_in_flight", 5), ("sequences_in_flight", -1), ("checkpoint_interval", -2),
                         ("timeout_probe_cycles", -1)]:
        o = _BitshiftOpts()
        setattr(o, field, value)
        # fake, never-dereferenced addresses: rejected before any CUDA call
        assert f(4096, 8192, 0.5, 16, 2, 8, 2, 12288, None, None, ctypes.pointer(o), 65536, 1 << 30, None) == INVALID


def test_dense_arguments_are_rejected_on_the_host(lib):
    INVALID, UNSUPPORTED, WORKSPACE = 1, 2, 3
    f = lib.bcjr_dense_forward
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_float] + [ctypes.c_int] * 3 + [ctypes.c_void_p] * 3 + \
        [ctypes.POINTER(_Opts), ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]

    def call(S=256, n=4, N=2, T=0.5, w=4096, c=8192, lam=12288, what=16384, ws=65536, opt=None):
        return f(w, c, lam, T, S, n, N, what, None, None, opt, ws, 1 << 20, None)

    assert call(T=0.0) == INVALID
    assert call(T=float("nan")) == INVALID
    assert call(n=0) == INVALID
    assert call(N=-1) == INVALID
    assert call(S=128) == UNSUPPORTED        # the dense kernels are built for 256 states
    assert call(w=0) == INVALID
    assert call(lam=0) == INVALID
    assert call(what=0) == INVALID
    assert call(ws=0) == WORKSPACE
    o = _Opts()
    o.checkpoint_interval = 4                 # the dense path keeps every step
    assert call(opt=ctypes.pointer(o)) == UNSUPPORTED
    o.checkpoint_interval = -1
    assert call(opt=ctypes.pointer(o)) == INVALID
    o.checkpoint_interval = 0
    o.sequences_in_flight = 1                 # only the automatic choice (0) is accepted
    assert call(opt=ctypes.pointer(o)) == INVALID
    assert call(N=0) == 0                     # nothing to do


def test_dense_lambda_arguments_are_rejected_on_the_host(lib):
    INVALID, UNSUPPORTED = 1, 2
    f = lib.bcjr_dense_backward_lambda
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p] * 5 + [ctypes.c_float] + [ctypes.c_int] * 3 + [ctypes.c_void_p] * 3 + \
        [ctypes.c_int, ctypes.POINTER(_Opts), ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]

    def call(S=256, n=4, N=2, T=0.5, g=4096, w=8192, c=12288, lam=16384, what=20480, gw=24576, gc=28672,
             gl=32768, ws=65536):
        return f(g, w, c, lam, what, T, S, n, N, gw, gc, gl, 0, None, ws, 1 << 20, None)

    assert call(gl=0) == INVALID              # the log-transition gradient is this call's output
    assert call(gl=32770) == INVALID          # misaligned
    assert call(T=-1.0) == INVALID
    assert call(S=64) == UNSUPPORTED
    assert call(g=0) == INVALID
    assert call(gc=0) == INVALID
