"""Comparison helpers for the GPU-vs-oracle parity tests.

Agreement criteria (fixed before any kernel was written): soft codewords and
marginals within 1e-5 absolute (codebook scale ~1); gradients within 1e-3
relative in L2; hard decode paths bit-exact.
"""
import numpy as np

W_HAT_ATOL = 1e-5
MARGINAL_ATOL = 1e-5
GRAD_REL_L2 = 1e-3
LOGZ_RTOL = 1e-5
# log Z is a sum of one log-sum-exp per step, each evaluated with the fast
# hardware 2^x and log2 (relative error of 2^x about 2^-22, absolute error of
# log2 about 2^-22.6, plus an fp32 sum of K terms): under 2^-21 natural-log
# units per step.  The bound is taken with a factor 2 margin and grows with the
# sequence length; where log Z is near zero only this absolute part applies.
LOGZ_ATOL_PER_STEP = 2.0 ** -20


def to_np(x):
    return x.detach().cpu().double().numpy() if hasattr(x, "detach") else np.asarray(x, dtype=np.float64)


def assert_abs(gpu, ref, atol, what):
    g, r = to_np(gpu), np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    assert np.isfinite(g).all(), f"{what}: non-finite values"
    err = np.abs(g - r).max() if g.size else 0.0
    assert err <= atol, f"{what}: max abs error {err:.3e} > {atol:.1e}"
    return err


def rel_l2(gpu, ref):
    g, r = to_np(gpu), np.asarray(ref, dtype=np.float64)
    return float(np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-300))


def assert_rel_l2(gpu, ref, tol, what):
    g = to_np(gpu)
    assert np.isfinite(g).all(), f"{what}: non-finite values"
    e = rel_l2(gpu, ref)
    assert e <= tol, f"{what}: relative L2 error {e:.3e} > {tol:.1e}"
    return e
