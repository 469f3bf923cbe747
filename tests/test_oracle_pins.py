"""Pins of the float64 oracle to things other than itself (CPU only).

Each test ties the oracle to a fact fixed by the paper's definitions or by the
mathematics ("BCJR-QAT", technical summary, "core mechanism": exact marginal
posteriors under the Boltzmann distribution over trellis paths; soft codeword
= Boltzmann expectation of the emitted codeword; exact gradients through the
trellis; T -> 0 recovers the hard Viterbi code; abstract: transfer-matrix
computation of a 1D Ising-like chain):

  * brute-force enumeration of every path (oracle/brute.py) -- marginals,
    soft codeword, log Z, and the VJP from the covariance identity;
  * central finite differences of the oracle's own soft codeword;
  * normalisation invariants (sum_s gamma_t = 1, log Z equal at every t);
  * closed forms: k = L (independent softmaxes), n = 1, T -> inf (uniform),
    constant codebook, the two-state tanh fixture (tests/golden), the
    translation identity sum grad_w + sum grad_c = sum g;
  * T -> 0: soft codeword -> codeword of the least-distortion path, and the
    max-sum decode equals the enumerated least-distortion path;
  * dense trellis: brute force, and T -> inf gives gamma_t = u P^t; the
    log-transition gradient against brute force and finite differences, and
    its entries sum to zero (a common shift of Lambda changes no path's
    probability).
"""
import os

import numpy as np
import pytest

import bcjr_inputs as I
import oracle
from oracle import brute

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")

# (state_bits, k, seq_len, T): k | L and k not dividing L, k = L, k = 1..4
TINY = [(4, 2, 4, 0.7), (4, 1, 5, 1.3), (5, 2, 3, 0.5), (3, 3, 3, 0.9), (6, 3, 3, 0.4),
        (5, 4, 2, 0.8), (6, 2, 4, 0.15), (2, 1, 6, 2.0)]


def _inputs(L, k, n, N=3, seed=0):
    S = 1 << L
    return (I.codebook(S, seed=100 + seed), I.weights(N, n, seed=200 + seed),
            I.upstream_grad(N, n, seed=300 + seed))


@pytest.mark.parametrize("L,k,n,T", TINY)
def test_forward_matches_path_enumeration(L, k, n, T):
    c, w, _ = _inputs(L, k, n, seed=L * 10 + k)
    w_hat, log_z, gamma = oracle.forward(w, c, T, L, k, want_gamma=True)
    b_what, b_lz, b_gamma = brute.forward(w, c, T, L, k)
    np.testing.assert_allclose(w_hat, b_what, rtol=0, atol=1e-12)
    np.testing.assert_allclose(log_z, b_lz, rtol=1e-13, atol=1e-12)
    np.testing.assert_allclose(gamma, b_gamma, rtol=0, atol=1e-13)


@pytest.mark.parametrize("L,k,n,T", TINY)
def test_backward_matches_covariance_identity(L, k, n, T):
    c, w, g = _inputs(L, k, n, seed=L * 10 + k + 1)
    grad_w, grad_c = oracle.backward(g, w, c, T, L, k)
    b_gw, b_gc = brute.backward(g, w, c, T, L, k)
    scale_w = np.abs(b_gw).max()
    scale_c = np.abs(b_gc).max()
    np.testing.assert_allclose(grad_w, b_gw, rtol=0, atol=1e-11 * max(scale_w, 1.0))
    np.testing.assert_allclose(grad_c, b_gc, rtol=0, atol=1e-11 * max(scale_c, 1.0))


def _five_point(f, x0, h):
    """f'(x0) by the five-point stencil at float32-representable points."""
    pts = np.array([x0 - 2 * h, x0 - h, x0 + h, x0 + 2 * h], dtype=np.float32).astype(np.float64)
    hh = (pts[2] - pts[1]) / 2.0  # exact spacing of the representable points
    assert abs(pts[3] - pts[0] - 4 * hh) < 1e-12
    v = [f(np.float32(p)) for p in pts]
    return (-v[3] + 8 * v[2] - 8 * v[1] + v[0]) / (12 * hh)


@pytest.mark.parametrize("L,k,n,T", [(8, 2, 12, 0.6), (7, 3, 9, 0.3), (9, 1, 10, 1.5)])
def test_backward_matches_finite_differences(L, k, n, T):
    c, w, g = _inputs(L, k, n, N=2, seed=7 + L)
    grad_w, grad_c = oracle.backward(g, w, c, T, L, k)
    g64 = g.double().numpy()

    def loss_w(i, u):
        def f(val):
            ww = w.clone()
            ww[i, u] = float(val)
            wh, _, _ = oracle.forward(ww, c, T, L, k)
            return float((g64 * wh).sum())
        return f

    def loss_c(r):
        def f(val):
            cc = c.clone()
            cc[r] = float(val)
            wh, _, _ = oracle.forward(w, cc, T, L, k)
            return float((g64 * wh).sum())
        return f

    h = 2.0 ** -9
    for (i, u) in [(0, 0), (0, n // 2), (1, n - 1)]:
        fd = _five_point(loss_w(i, u), float(w[i, u]), h)
        assert abs(fd - grad_w[i, u]) <= 1e-7 * max(1.0, abs(grad_w).max()), (i, u, fd, grad_w[i, u])
    rng = np.random.default_rng(L)
    for r in rng.choice(1 << L, size=4, replace=False):
        fd = _five_point(loss_c(int(r)), float(c[r]), h)
        assert abs(fd - grad_c[r]) <= 1e-7 * max(1.0, abs(grad_c).max()), (r, fd, grad_c[r])


@pytest.mark.parametrize("L,k,T", [(8, 2, 0.5), (8, 3, 0.2), (7, 1, 1.0)])
def test_normalisation_invariants(L, k, T):
    c, w, _ = _inputs(L, k, 20, N=1, seed=3)
    alpha, beta = oracle.alpha_beta(w[0], c, T, L, k)
    lz_t = np.array([np.logaddexp.reduce(alpha[t] + beta[t]) for t in range(alpha.shape[0])])
    np.testing.assert_allclose(lz_t, lz_t[-1], rtol=0, atol=1e-10)
    _, log_z, gamma = oracle.forward(w, c, T, L, k, want_gamma=True)
    np.testing.assert_allclose(log_z[0], lz_t[-1], rtol=0, atol=1e-10)
    np.testing.assert_allclose(gamma.sum(axis=2), 1.0, rtol=0, atol=1e-12)
    assert (gamma >= 0).all()


def _softmax(x):
    e = np.exp(x - x.max(axis=-1, keepdims=True))
    return e / e.sum(axis=-1, keepdims=True)


@pytest.mark.parametrize("L,n,T", [(3, 5, 0.7), (5, 4, 0.3), (1, 6, 1.0)])
def test_k_equals_L_factorises_into_softmaxes(L, n, T):
    # k = L: pred(s) is every state, so the chain factorises over steps.
    c, w, g = _inputs(L, L, n, N=2, seed=11)
    c64, w64, g64 = (x.double().numpy() for x in (c, w, g))
    phi = -((w64[:, :, None] - c64[None, None, :]) ** 2) / T
    gam = _softmax(phi)
    w_hat_cf = (gam * c64).sum(axis=2)
    var_cf = (gam * c64 ** 2).sum(axis=2) - w_hat_cf ** 2
    gw_cf = (2.0 / T) * g64 * var_cf
    gc_cf = (g64[:, :, None] * gam * (1.0 + (2.0 / T) * (c64[None, None, :] - w_hat_cf[:, :, None])
                                       * (w64[:, :, None] - c64[None, None, :]))).sum(axis=(0, 1))
    w_hat, _, gamma = oracle.forward(w, c, T, L, L, want_gamma=True)
    grad_w, grad_c = oracle.backward(g, w, c, T, L, L)
    np.testing.assert_allclose(gamma, gam, rtol=0, atol=1e-13)
    np.testing.assert_allclose(w_hat, w_hat_cf, rtol=0, atol=1e-13)
    np.testing.assert_allclose(grad_w, gw_cf, rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(grad_c, gc_cf, rtol=1e-11, atol=1e-11)


@pytest.mark.parametrize("L,k", [(8, 2), (6, 3)])
def test_single_step_is_a_softmax(L, k):
    c, w, _ = _inputs(L, k, 1, N=4, seed=12)
    T = 0.37
    phi = -((w.double().numpy()[:, :, None] - c.double().numpy()[None, None, :]) ** 2) / T
    _, log_z, gamma = oracle.forward(w, c, T, L, k, want_gamma=True)
    np.testing.assert_allclose(gamma, _softmax(phi), rtol=0, atol=1e-14)
    np.testing.assert_allclose(log_z, np.logaddexp.reduce(phi[:, 0, :], axis=1), rtol=1e-14)


def test_infinite_temperature_is_uniform():
    L, k, n = 8, 2, 10
    c, w, _ = _inputs(L, k, n, N=2, seed=13)
    w_hat, _, gamma = oracle.forward(w, c, 1e12, L, k, want_gamma=True)
    np.testing.assert_allclose(gamma, 1.0 / (1 << L), rtol=1e-9)
    np.testing.assert_allclose(w_hat, c.double().mean().item(), rtol=0, atol=1e-9)


def test_constant_codebook():
    L, k, n, T = 7, 2, 9, 0.25
    c = np.full(1 << L, 0.625, dtype=np.float32)
    _, w, g = _inputs(L, k, n, N=2, seed=14)
    w_hat, _, gamma = oracle.forward(w, c, T, L, k, want_gamma=True)
    grad_w, grad_c = oracle.backward(g, w, c, T, L, k)
    np.testing.assert_allclose(w_hat, 0.625, rtol=0, atol=1e-14)
    np.testing.assert_allclose(gamma, 1.0 / (1 << L), rtol=1e-12)
    np.testing.assert_allclose(grad_w, 0.0, atol=1e-12)
    # Every state is equally likely, so dL/dc(r) = sum_u g_u / S + (2/T) sum_u (w_u - c) * 0.
    np.testing.assert_allclose(grad_c, g.double().sum().item() / (1 << L), rtol=1e-10)


def test_two_state_tanh_fixture():
    rows = [list(map(float, ln.split())) for ln in open(os.path.join(GOLDEN, "two_state_tanh.txt"))
            if ln.strip() and not ln.lstrip().startswith("#")]
    c = np.array([-1.0, 1.0], dtype=np.float32)
    for T, w, w_hat_ref, dwhat_ref in rows:
        wt = np.array([[w]], dtype=np.float32)
        w_hat, _, _ = oracle.forward(wt, c, T, 1, 1)
        grad_w, _ = oracle.backward(np.ones((1, 1), np.float32), wt, c, T, 1, 1)
        assert abs(w_hat[0, 0] - w_hat_ref) < 1e-14
        assert abs(grad_w[0, 0] - dwhat_ref) < 1e-13


@pytest.mark.parametrize("L,k,n,T", [(10, 2, 16, 0.2), (9, 3, 12, 0.05), (8, 4, 10, 1.0)])
def test_translation_identity(L, k, n, T):
    # Shifting w and c by the same delta shifts w_hat by delta and leaves the
    # path distribution unchanged, so sum_u dL/dw_u + sum_r dL/dc(r) = sum_u g_u.
    c, w, g = _inputs(L, k, n, N=3, seed=15)
    grad_w, grad_c = oracle.backward(g, w, c, T, L, k)
    total = grad_w.sum() + grad_c.sum()
    assert abs(total - g.double().sum().item()) < 1e-9 * max(1.0, np.abs(grad_w).sum())


@pytest.mark.parametrize("L,k,n", [(4, 2, 5), (5, 1, 7), (6, 2, 5), (6, 3, 4), (5, 2, 6)])
def test_hard_decode_is_least_distortion_path(L, k, n):
    c, w, _ = _inputs(L, k, n, N=6, seed=16)
    states, w_hard, metric = oracle.viterbi(w, c, L, k)
    paths, dist, gap = brute.min_distortion_paths(w, c, L, k)
    assert (gap > 1e-9).all()  # continuous inputs: no ties
    np.testing.assert_array_equal(states, paths)
    np.testing.assert_allclose(-metric, dist, rtol=1e-13)
    np.testing.assert_array_equal(w_hard, c.numpy()[paths])


@pytest.mark.parametrize("L,k,n", [(4, 2, 5), (6, 2, 5), (5, 3, 4)])
def test_zero_temperature_limit(L, k, n):
    # error of w_hat vs c(s*) is at most (#paths) exp(-gap / T) max|c|
    c, w, _ = _inputs(L, k, n, N=4, seed=17)
    paths, _, gap = brute.min_distortion_paths(w, c, L, k)
    n_paths = (1 << L) * (1 << k) ** (n - 1)
    T = float(gap.min()) / 80.0
    w_hat, log_z, _ = oracle.forward(w, c, T, L, k)
    cmax = np.abs(c.numpy()).max()
    bound = n_paths * np.exp(-80.0) * cmax
    # float64 rounding: alpha, beta and log Z are ~|log Z| large, so each
    # exp(alpha + beta - log Z) carries a relative error of a few eps * |log Z|.
    rounding = 16 * np.finfo(np.float64).eps * np.abs(log_z).max() * cmax
    np.testing.assert_allclose(w_hat, c.numpy()[paths], rtol=0, atol=bound + rounding)


def test_dense_matches_path_enumeration():
    S, n, T = 4, 5, 0.6
    lam = I.log_transition(S, seed=21)
    c = I.codebook(S, seed=22)
    w = I.weights(2, n, seed=23)
    g = I.upstream_grad(2, n, seed=24)
    a = oracle.dense_forward(w, c, lam, T, want_gamma=True)
    b = brute.dense_forward(w, c, lam, T)
    for x, y in zip(a, b):
        np.testing.assert_allclose(x, y, rtol=1e-13, atol=1e-13)
    ga = oracle.dense_backward(g, w, c, lam, T, want_grad_lam=True)
    gb = brute.dense_backward(g, w, c, lam, T)
    assert len(ga) == len(gb) == 3
    for x, y in zip(ga, gb):
        np.testing.assert_allclose(x, y, rtol=1e-11, atol=1e-12)


def test_dense_transition_gradient_matches_finite_differences():
    S, n, T = 8, 6, 0.5
    lam = I.log_transition(S, seed=31)
    c = I.codebook(S, seed=32)
    w = I.weights(2, n, seed=33)
    g = I.upstream_grad(2, n, seed=34)
    _, _, grad_lam = oracle.dense_backward(g, w, c, lam, T, want_grad_lam=True)
    g64 = g.double().numpy()

    def loss(p, r):
        def f(val):
            ll = lam.clone()
            ll[p, r] = float(val)
            return float((g64 * oracle.dense_forward(w, c, ll, T)[0]).sum())
        return f

    h = 2.0 ** -9
    scale = max(1.0, np.abs(grad_lam).max())
    for (p, r) in [(0, 0), (3, 5), (7, 1), (5, 5), (2, 7)]:
        fd = _five_point(loss(p, r), float(lam[p, r]), h)
        assert abs(fd - grad_lam[p, r]) <= 1e-7 * scale, (p, r, fd, grad_lam[p, r])


def test_dense_transition_gradient_sums_to_zero():
    # Adding one constant to every Lambda entry adds (n-1) times it to every
    # path's log-weight, which leaves the path distribution unchanged.
    S, n, T = 16, 9, 0.3
    lam = I.log_transition(S, seed=35)
    c = I.codebook(S, seed=36)
    w = I.weights(3, n, seed=37)
    g = I.upstream_grad(3, n, seed=38)
    _, _, grad_lam = oracle.dense_backward(g, w, c, lam, T, want_grad_lam=True)
    assert abs(grad_lam.sum()) <= 1e-12 * max(1.0, np.abs(grad_lam).sum())
    assert np.abs(grad_lam).max() > 1e-3


def test_dense_infinite_temperature_is_a_markov_chain():
    # T -> inf: emissions vanish, gamma_t = u P^t with u uniform and P = exp(Lam)
    S, n = 8, 6
    lam = I.log_transition(S, seed=25)
    c = I.codebook(S, seed=26)
    w = I.weights(1, n, seed=27)
    _, _, gamma = oracle.dense_forward(w, c, lam, 1e13, want_gamma=True)
    P = np.exp(lam.double().numpy())
    u = np.full(S, 1.0 / S)
    for t in range(n):
        np.testing.assert_allclose(gamma[0, t], u @ np.linalg.matrix_power(P, t), rtol=1e-6, atol=1e-9)


def test_dense_with_uniform_transitions_equals_k_equals_L():
    # Lam = -log S everywhere is the k = L bitshift trellis (uniform transitions).
    L, n, T = 3, 5, 0.45
    S = 1 << L
    lam = np.full((S, S), -np.log(S), dtype=np.float32)
    c, w, g = _inputs(L, L, n, N=2, seed=28)
    a = oracle.dense_forward(w, c, lam, T)[0]
    b = oracle.forward(w, c, T, L, L)[0]
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-13)
    np.testing.assert_allclose(oracle.dense_backward(g, w, c, lam, T)[0],
                               oracle.backward(g, w, c, T, L, L)[0], rtol=1e-11, atol=1e-12)
