/*
 * bcjr_oracle.c -- plain, slow float64 CPU oracle for BCJR-QAT.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file: only the tests, the package's smoke check and the
 * benchmark's CPU-baseline leg use it.  It shares no code, header, table or
 * helper with the CUDA library.
 *
 * What it computes ("BCJR-QAT: A Differentiable Relaxation of Trellis-Coded
 * Weight Quantization", abstract and technical summary, "core mechanism"):
 * the trellis is read as a chain whose paths carry Boltzmann weights at
 * temperature T; the BCJR forward-backward sum-product gives the exact
 * marginal posterior of every state, and the soft codeword is the Boltzmann
 * expectation of the emitted codeword,
 *
 *     w_hat_t = sum_s c(s) p_T(s_t = s | w).
 *
 * The soft codeword is differentiable in the weight preimage w and in the
 * trellis parameters (the codebook c); the backward entry points give that
 * vector-Jacobian product.  As T -> 0 the soft codeword becomes the hard
 * Viterbi decode, which oracle_viterbi computes by plain max-sum.
 *
 * Readings of what the pages leave open (each one is also listed in the
 * design notes):
 *   - emission log-weight   phi_t(s) = -(w_t - c(s))^2 / T, one weight per step;
 *   - bitshift trellis      pred(s) = { (j << (L-k)) | (s >> k) : 0 <= j < 2^k },
 *                           succ(p) = { ((p << k) & (S-1)) | b : 0 <= b < 2^k };
 *   - uniform initial state, free end (beta_{n-1} = 0);
 *   - log_z is the natural log of the sum over all paths of exp(sum_t phi_t)
 *     (the constant 1/S of the uniform prior is left out);
 *   - dense trellis: path log-weight adds Lambda[s_{t-1}][s_t] for t >= 1,
 *     Lambda[i][j] with i the source state.
 *
 * Every recursion below is the unfactored textbook form: one log-sum-exp over
 * the 2^k predecessors (or successors) of EVERY state, natural logarithms,
 * float64 arithmetic, no rescaling beyond the max-subtraction inside each
 * log-sum-exp.  All arrays are row-major and contiguous.
 *
 * Build:  gcc -O2 -fopenmp -ffp-contract=off -fPIC -shared -o liboracle.so bcjr_oracle.c -lm
 * (-ffp-contract=off keeps every multiply and add separately rounded, which
 * the max-sum metric below relies on to be reproducible bit for bit.)
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_BAD_ARG 1
#define ORACLE_NO_MEMORY 2

/* log(sum_i exp(x[i])) with the max subtracted first. */
static double log_sum_exp(const double* x, int m) {
  double mx = -INFINITY;
  for (int i = 0; i < m; ++i)
    if (x[i] > mx) mx = x[i];
  if (mx == -INFINITY) return -INFINITY;
  double s = 0.0;
  for (int i = 0; i < m; ++i) s += exp(x[i] - mx);
  return mx + log(s);
}

static int bitshift_args_ok(int L, int k, int n, int N, double T) {
  return L >= 1 && L <= 20 && k >= 1 && k <= L && n >= 1 && N >= 0 && T > 0.0 && isfinite(T);
}

/* Predecessor j of state s:  (j << (L-k)) | (s >> k). */
static inline int pred_state(int s, int j, int L, int k) { return (j << (L - k)) | (s >> k); }
/* Successor b of state p:   ((p << k) & (S-1)) | b. */
static inline int succ_state(int p, int b, int L, int k) { return ((p << k) & ((1 << L) - 1)) | b; }

/* phi_t(s) = -(w_t - c(s))^2 / T */
static inline double emission(float w, float c, double T) {
  double d = (double)w - (double)c;
  return -(d * d) / T;
}

/* ---------------------------------------------------------------------------
 * Forward recursion over the bitshift trellis, one sequence:
 *   alpha_0(s) = phi_0(s)
 *   alpha_t(s) = phi_t(s) + LSE_{p in pred(s)} alpha_{t-1}(p)
 * alpha is [n][S].
 * ------------------------------------------------------------------------- */
static void bitshift_alpha(const float* w, const float* c, double T, int L, int k, int n,
                           double* alpha) {
  const int S = 1 << L, K = 1 << k;
  double terms[64];
  double* x = K <= 64 ? terms : (double*)malloc(sizeof(double) * K);
  for (int s = 0; s < S; ++s) alpha[s] = emission(w[0], c[s], T);
  for (int t = 1; t < n; ++t) {
    const double* prev = alpha + (size_t)(t - 1) * S;
    double* cur = alpha + (size_t)t * S;
    for (int s = 0; s < S; ++s) {
      for (int j = 0; j < K; ++j) x[j] = prev[pred_state(s, j, L, k)];
      cur[s] = emission(w[t], c[s], T) + log_sum_exp(x, K);
    }
  }
  if (x != terms) free(x);
}

/* One backward step:  beta_t(p) = LSE_{s in succ(p)} [phi_{t+1}(s) + beta_{t+1}(s)]. */
static void bitshift_beta_step(const float* w, const float* c, double T, int L, int k, int t,
                               const double* beta_next, double* beta_t) {
  const int S = 1 << L, K = 1 << k;
  double terms[64];
  double* x = K <= 64 ? terms : (double*)malloc(sizeof(double) * K);
  for (int p = 0; p < S; ++p) {
    for (int b = 0; b < K; ++b) {
      int s = succ_state(p, b, L, k);
      x[b] = emission(w[t + 1], c[s], T) + beta_next[s];
    }
    beta_t[p] = log_sum_exp(x, K);
  }
  if (x != terms) free(x);
}

/* alpha [n][S] and beta [n][S] of one sequence (for invariant checks). */
int oracle_alpha_beta(const float* w, const float* c, double T, int L, int k, int n,
                      double* alpha, double* beta) {
  if (!bitshift_args_ok(L, k, n, 1, T) || !w || !c || !alpha || !beta) return ORACLE_BAD_ARG;
  const int S = 1 << L;
  bitshift_alpha(w, c, T, L, k, n, alpha);
  for (int s = 0; s < S; ++s) beta[(size_t)(n - 1) * S + s] = 0.0;
  for (int t = n - 2; t >= 0; --t)
    bitshift_beta_step(w, c, T, L, k, t, beta + (size_t)(t + 1) * S, beta + (size_t)t * S);
  return ORACLE_OK;
}

/* ---------------------------------------------------------------------------
 * Soft codeword (forward call), N independent sequences.
 *   log_z       = LSE_s alpha_{n-1}(s)
 *   gamma_t(s)  = exp(alpha_t(s) + beta_t(s) - log_z)
 *   w_hat_t     = sum_s c(s) gamma_t(s)
 * w_hat [N][n]; gamma [N][n][S] or NULL; log_z [N] or NULL.
 * The beta pass runs from t = n-1 down to 0 and combines with the stored
 * alpha at each t, as the forward-backward algorithm does.
 * ------------------------------------------------------------------------- */
int oracle_forward(const float* w, const float* c, double T, int L, int k, int n, int N,
                   double* w_hat, double* gamma, double* log_z, int nthreads) {
  if (!bitshift_args_ok(L, k, n, N, T) || !w || !c || !w_hat) return ORACLE_BAD_ARG;
  const int S = 1 << L;
  int status = ORACLE_OK;
#ifdef _OPENMP
  if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
#endif
  for (int q = 0; q < N; ++q) {
    const float* wq = w + (size_t)q * n;
    double* alpha = (double*)malloc(sizeof(double) * (size_t)n * S);
    double* beta_a = (double*)malloc(sizeof(double) * S);
    double* beta_b = (double*)malloc(sizeof(double) * S);
    if (!alpha || !beta_a || !beta_b) {
      status = ORACLE_NO_MEMORY;
      free(alpha); free(beta_a); free(beta_b);
      continue;
    }
    bitshift_alpha(wq, c, T, L, k, n, alpha);
    const double lz = log_sum_exp(alpha + (size_t)(n - 1) * S, S);
    if (log_z) log_z[q] = lz;
    double* beta_t = beta_a;
    double* beta_next = beta_b;
    for (int s = 0; s < S; ++s) beta_t[s] = 0.0;
    for (int t = n - 1; t >= 0; --t) {
      if (t < n - 1) {
        double* tmp = beta_next; beta_next = beta_t; beta_t = tmp;
        bitshift_beta_step(wq, c, T, L, k, t, beta_next, beta_t);
      }
      double acc = 0.0;
      for (int s = 0; s < S; ++s) {
        double g = exp(alpha[(size_t)t * S + s] + beta_t[s] - lz);
        if (gamma) gamma[((size_t)q * n + t) * S + s] = g;
        acc += (double)c[s] * g;
      }
      w_hat[(size_t)q * n + t] = acc;
    }
    free(alpha); free(beta_a); free(beta_b);
  }
  return status;
}

/* ---------------------------------------------------------------------------
 * Vector-Jacobian product (backward call).
 *
 * With G = sum_t g_t c(s_t) along a path, L = sum_t g_t w_hat_t = E[G], and
 * the path log-weight E = sum_t phi_t(s_t):
 *   dL/dw_u    = Cov(G, dE/dw_u)    = (2/T) Cov(G, c(s_u))
 *   dL/dc(r)   = E[dG/dc(r)] + Cov(G, dE/dc(r))
 *              = sum_u g_u gamma_u(r) + (2/T) sum_u (w_u - c(r)) Cov(G, 1[s_u = r]).
 * Both covariances are psi_u(r) = E[(G - E G) 1[s_u = r]], which the
 * forward-backward recursions give as
 *   psi_u(r) = gamma_u(r) (F_u(r) + e_u(r) + B_u(r)),   e_t(s) = g_t (c(s) - w_hat_t),
 *   F_u(r)   = E[sum_{t<u} e_t(s_t) | s_u = r]
 *            = sum_{p in pred(r)} pi(p|r) (F_{u-1}(p) + e_{u-1}(p)),
 *              pi(p|r) = exp(alpha_{u-1}(p) - LSE_{p' in pred(r)} alpha_{u-1}(p')),  F_0 = 0,
 *   B_u(r)   = E[sum_{t>u} e_t(s_t) | s_u = r]
 *            = sum_{s in succ(r)} rho(s|r) (e_{u+1}(s) + B_{u+1}(s)),
 *              rho(s|r) = exp(phi_{u+1}(s) + beta_{u+1}(s) - beta_u(r)),        B_{n-1} = 0.
 * Then dL/dw_u = (2/T) sum_r psi_u(r) c(r) and
 *      dL/dc(r) = sum_u [g_u gamma_u(r) + (2/T) psi_u(r) (w_u - c(r))],
 * summed over all sequences.
 * grad_w [N][n]; grad_c [S] (overwritten).  w_hat is recomputed here.
 * ------------------------------------------------------------------------- */
int oracle_backward(const float* g, const float* w, const float* c, double T, int L, int k, int n,
                    int N, double* grad_w, double* grad_c, int nthreads) {
  if (!bitshift_args_ok(L, k, n, N, T) || !g || !w || !c || !grad_w || !grad_c)
    return ORACLE_BAD_ARG;
  const int S = 1 << L, K = 1 << k;
  int status = ORACLE_OK;
  double* gc_seq = (double*)calloc((size_t)(N > 0 ? N : 1) * S, sizeof(double));
  if (!gc_seq) return ORACLE_NO_MEMORY;
#ifdef _OPENMP
  if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
#endif
  for (int q = 0; q < N; ++q) {
    const float* wq = w + (size_t)q * n;
    const float* gq = g + (size_t)q * n;
    double* gcq = gc_seq + (size_t)q * S;
    double* alpha = (double*)malloc(sizeof(double) * (size_t)n * S);
    double* F = (double*)malloc(sizeof(double) * (size_t)n * S);
    double* beta_t = (double*)malloc(sizeof(double) * S);
    double* beta_next = (double*)malloc(sizeof(double) * S);
    double* B_t = (double*)malloc(sizeof(double) * S);
    double* B_next = (double*)malloc(sizeof(double) * S);
    double* what = (double*)malloc(sizeof(double) * n);
    double* x = (double*)malloc(sizeof(double) * K);
    if (!alpha || !F || !beta_t || !beta_next || !B_t || !B_next || !what || !x) {
      status = ORACLE_NO_MEMORY;
      free(alpha); free(F); free(beta_t); free(beta_next); free(B_t); free(B_next);
      free(what); free(x);
      continue;
    }
    bitshift_alpha(wq, c, T, L, k, n, alpha);
    const double lz = log_sum_exp(alpha + (size_t)(n - 1) * S, S);

    /* First backward pass: the soft codeword w_hat_t (needed to centre e_t). */
    for (int s = 0; s < S; ++s) beta_t[s] = 0.0;
    for (int t = n - 1; t >= 0; --t) {
      if (t < n - 1) {
        double* tmp = beta_next; beta_next = beta_t; beta_t = tmp;
        bitshift_beta_step(wq, c, T, L, k, t, beta_next, beta_t);
      }
      double acc = 0.0;
      for (int s = 0; s < S; ++s) acc += (double)c[s] * exp(alpha[(size_t)t * S + s] + beta_t[s] - lz);
      what[t] = acc;
    }

    /* Forward accumulator F. */
    for (int s = 0; s < S; ++s) F[s] = 0.0;
    for (int u = 1; u < n; ++u) {
      const double* ap = alpha + (size_t)(u - 1) * S;
      const double* Fp = F + (size_t)(u - 1) * S;
      double* Fu = F + (size_t)u * S;
      for (int r = 0; r < S; ++r) {
        for (int j = 0; j < K; ++j) x[j] = ap[pred_state(r, j, L, k)];
        const double lse = log_sum_exp(x, K);
        double acc = 0.0;
        for (int j = 0; j < K; ++j) {
          const int p = pred_state(r, j, L, k);
          const double pi = exp(ap[p] - lse);
          const double e_prev = (double)gq[u - 1] * ((double)c[p] - what[u - 1]);
          acc += pi * (Fp[p] + e_prev);
        }
        Fu[r] = acc;
      }
    }

    /* Second backward pass: beta, B, psi and the gradients. */
    for (int s = 0; s < S; ++s) { beta_t[s] = 0.0; B_t[s] = 0.0; }
    for (int u = n - 1; u >= 0; --u) {
      if (u < n - 1) {
        double* tmp = beta_next; beta_next = beta_t; beta_t = tmp;
        tmp = B_next; B_next = B_t; B_t = tmp;
        bitshift_beta_step(wq, c, T, L, k, u, beta_next, beta_t);
        for (int r = 0; r < S; ++r) {
          double acc = 0.0;
          for (int b = 0; b < K; ++b) {
            const int s = succ_state(r, b, L, k);
            const double rho = exp(emission(wq[u + 1], c[s], T) + beta_next[s] - beta_t[r]);
            const double e_next = (double)gq[u + 1] * ((double)c[s] - what[u + 1]);
            acc += rho * (e_next + B_next[s]);
          }
          B_t[r] = acc;
        }
      }
      double gw = 0.0;
      for (int r = 0; r < S; ++r) {
        const double gm = exp(alpha[(size_t)u * S + r] + beta_t[r] - lz);
        const double e_u = (double)gq[u] * ((double)c[r] - what[u]);
        const double psi = gm * (F[(size_t)u * S + r] + e_u + B_t[r]);
        gw += psi * (double)c[r];
        gcq[r] += (double)gq[u] * gm + (2.0 / T) * psi * ((double)wq[u] - (double)c[r]);
      }
      grad_w[(size_t)q * n + u] = (2.0 / T) * gw;
    }
    free(alpha); free(F); free(beta_t); free(beta_next); free(B_t); free(B_next);
    free(what); free(x);
  }
  /* Sum the per-sequence codebook gradients in sequence order. */
  for (int s = 0; s < S; ++s) grad_c[s] = 0.0;
  for (int q = 0; q < N; ++q)
    for (int s = 0; s < S; ++s) grad_c[s] += gc_seq[(size_t)q * S + s];
  free(gc_seq);
  return status;
}

/* ---------------------------------------------------------------------------
 * Hard decode (the T -> 0 limit): the path of least total distortion.
 *   D_0(s) = -(w_0 - c(s))^2
 *   D_t(s) = -(w_t - c(s))^2 + max_{p in pred(s)} D_{t-1}(p)
 * with every difference, square and sum rounded separately in float64.
 * Ties: the lowest j among equal predecessors, the lowest s at the end.
 * states [N][n] (int32), w_hard [N][n] (= c(s_t)), metric [N] (the best D_{n-1}) or NULL.
 * ------------------------------------------------------------------------- */
int oracle_viterbi(const float* w, const float* c, int L, int k, int n, int N, int32_t* states,
                   float* w_hard, double* metric, int nthreads) {
  if (!bitshift_args_ok(L, k, n, N, 1.0) || !w || !c || !states) return ORACLE_BAD_ARG;
  const int S = 1 << L, K = 1 << k;
  int status = ORACLE_OK;
#ifdef _OPENMP
  if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
#endif
  for (int q = 0; q < N; ++q) {
    const float* wq = w + (size_t)q * n;
    double* D_prev = (double*)malloc(sizeof(double) * S);
    double* D_cur = (double*)malloc(sizeof(double) * S);
    unsigned char* bp = (unsigned char*)malloc((size_t)n * S);
    if (!D_prev || !D_cur || !bp) {
      status = ORACLE_NO_MEMORY;
      free(D_prev); free(D_cur); free(bp);
      continue;
    }
    for (int s = 0; s < S; ++s) {
      double d = (double)wq[0] - (double)c[s];
      double sq = d * d;
      D_cur[s] = -sq;
    }
    for (int t = 1; t < n; ++t) {
      double* tmp = D_prev; D_prev = D_cur; D_cur = tmp;
      for (int s = 0; s < S; ++s) {
        int best_j = 0;
        double best = D_prev[pred_state(s, 0, L, k)];
        for (int j = 1; j < K; ++j) {
          double v = D_prev[pred_state(s, j, L, k)];
          if (v > best) { best = v; best_j = j; }
        }
        double d = (double)wq[t] - (double)c[s];
        double sq = d * d;
        D_cur[s] = best + (-sq);
        bp[(size_t)t * S + s] = (unsigned char)best_j;
      }
    }
    int s_end = 0;
    for (int s = 1; s < S; ++s)
      if (D_cur[s] > D_cur[s_end]) s_end = s;
    if (metric) metric[q] = D_cur[s_end];
    int32_t* st = states + (size_t)q * n;
    st[n - 1] = s_end;
    for (int t = n - 1; t >= 1; --t) st[t - 1] = pred_state(st[t], bp[(size_t)t * S + st[t]], L, k);
    if (w_hard)
      for (int t = 0; t < n; ++t) w_hard[(size_t)q * n + t] = c[st[t]];
    free(D_prev); free(D_cur); free(bp);
  }
  return status;
}

/* ---------------------------------------------------------------------------
 * Dense (fully connected) trellis: the transfer-matrix form of the abstract.
 *   alpha_0(s) = phi_0(s)
 *   alpha_t(s) = phi_t(s) + LSE_p [alpha_{t-1}(p) + Lam[p][s]]
 *   beta_{n-1} = 0,  beta_t(p) = LSE_s [Lam[p][s] + phi_{t+1}(s) + beta_{t+1}(s)]
 * Lam is [S][S], row = source state.  Same outputs as the bitshift calls.
 * ------------------------------------------------------------------------- */
static void dense_alpha(const float* w, const float* c, const float* lam, double T, int S, int n,
                        double* alpha, double* x) {
  for (int s = 0; s < S; ++s) alpha[s] = emission(w[0], c[s], T);
  for (int t = 1; t < n; ++t) {
    const double* prev = alpha + (size_t)(t - 1) * S;
    double* cur = alpha + (size_t)t * S;
    for (int s = 0; s < S; ++s) {
      for (int p = 0; p < S; ++p) x[p] = prev[p] + (double)lam[(size_t)p * S + s];
      cur[s] = emission(w[t], c[s], T) + log_sum_exp(x, S);
    }
  }
}

static void dense_beta_step(const float* w, const float* c, const float* lam, double T, int S,
                            int t, const double* beta_next, double* beta_t, double* x) {
  for (int p = 0; p < S; ++p) {
    for (int s = 0; s < S; ++s)
      x[s] = (double)lam[(size_t)p * S + s] + emission(w[t + 1], c[s], T) + beta_next[s];
    beta_t[p] = log_sum_exp(x, S);
  }
}

static int dense_args_ok(int S, int n, int N, double T) {
  return S >= 1 && S <= 4096 && n >= 1 && N >= 0 && T > 0.0 && isfinite(T);
}

int oracle_dense_forward(const float* w, const float* c, const float* lam, double T, int S, int n,
                         int N, double* w_hat, double* gamma, double* log_z, int nthreads) {
  if (!dense_args_ok(S, n, N, T) || !w || !c || !lam || !w_hat) return ORACLE_BAD_ARG;
  int status = ORACLE_OK;
#ifdef _OPENMP
  if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
#endif
  for (int q = 0; q < N; ++q) {
    const float* wq = w + (size_t)q * n;
    double* alpha = (double*)malloc(sizeof(double) * (size_t)n * S);
    double* beta_t = (double*)malloc(sizeof(double) * S);
    double* beta_next = (double*)malloc(sizeof(double) * S);
    double* x = (double*)malloc(sizeof(double) * S);
    if (!alpha || !beta_t || !beta_next || !x) {
      status = ORACLE_NO_MEMORY;
      free(alpha); free(beta_t); free(beta_next); free(x);
      continue;
    }
    dense_alpha(wq, c, lam, T, S, n, alpha, x);
    const double lz = log_sum_exp(alpha + (size_t)(n - 1) * S, S);
    if (log_z) log_z[q] = lz;
    for (int s = 0; s < S; ++s) beta_t[s] = 0.0;
    for (int t = n - 1; t >= 0; --t) {
      if (t < n - 1) {
        double* tmp = beta_next; beta_next = beta_t; beta_t = tmp;
        dense_beta_step(wq, c, lam, T, S, t, beta_next, beta_t, x);
      }
      double acc = 0.0;
      for (int s = 0; s < S; ++s) {
        double gm = exp(alpha[(size_t)t * S + s] + beta_t[s] - lz);
        if (gamma) gamma[((size_t)q * n + t) * S + s] = gm;
        acc += (double)c[s] * gm;
      }
      w_hat[(size_t)q * n + t] = acc;
    }
    free(alpha); free(beta_t); free(beta_next); free(x);
  }
  return status;
}

/* Dense VJP: the same psi/F/B formulas with pred(r) = succ(p) = all states and
 * pi(p|r) = exp(alpha_{u-1}(p) + Lam[p][r] - LSE_p'[alpha_{u-1}(p') + Lam[p'][r]]),
 * rho(s|r) = exp(Lam[r][s] + phi_{u+1}(s) + beta_{u+1}(s) - beta_u(r)).
 *
 * grad_lam (optional, [S][S]): the gradient with respect to the log-transitions
 * ("key technical innovations": exact gradients with respect to the trellis
 * parameters).  Lam[p][r] enters the path log-weight once per transition
 * p -> r, so dL/dLam[p][r] = Cov(G, #transitions p -> r) with
 * G = sum_u g_u c(s_u), i.e. summed over the transitions u-1 -> u,
 *   xi_u(p,r) = P(s_{u-1} = p, s_u = r)
 *             = exp(alpha_{u-1}(p) + Lam[p][r] + phi_u(r) + beta_u(r) - log Z),
 *   dL/dLam[p][r] = sum_u xi_u(p,r) (F_{u-1}(p) + e_{u-1}(p) + e_u(r) + B_u(r)),
 * where e_u(r) = g_u (c(r) - w_hat_u) and F, B are the conditional expectations
 * of the past and future parts of G - E[G] defined above (the Markov property
 * splits E[G - E[G] | s_{u-1} = p, s_u = r] into those two parts). */
int oracle_dense_backward(const float* g, const float* w, const float* c, const float* lam,
                          double T, int S, int n, int N, double* grad_w, double* grad_c,
                          double* grad_lam, int nthreads) {
  if (!dense_args_ok(S, n, N, T) || !g || !w || !c || !lam || !grad_w || !grad_c)
    return ORACLE_BAD_ARG;
  int status = ORACLE_OK;
  double* gc_seq = (double*)calloc((size_t)(N > 0 ? N : 1) * S, sizeof(double));
  double* gl_seq = grad_lam ? (double*)calloc((size_t)(N > 0 ? N : 1) * S * S, sizeof(double)) : NULL;
  if (!gc_seq || (grad_lam && !gl_seq)) {
    free(gc_seq);
    free(gl_seq);
    return ORACLE_NO_MEMORY;
  }
#ifdef _OPENMP
  if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
#endif
  for (int q = 0; q < N; ++q) {
    const float* wq = w + (size_t)q * n;
    const float* gq = g + (size_t)q * n;
    double* gcq = gc_seq + (size_t)q * S;
    double* glq = gl_seq ? gl_seq + (size_t)q * S * S : NULL;
    double* alpha = (double*)malloc(sizeof(double) * (size_t)n * S);
    double* F = (double*)malloc(sizeof(double) * (size_t)n * S);
    double* beta_t = (double*)malloc(sizeof(double) * S);
    double* beta_next = (double*)malloc(sizeof(double) * S);
    double* B_t = (double*)malloc(sizeof(double) * S);
    double* B_next = (double*)malloc(sizeof(double) * S);
    double* what = (double*)malloc(sizeof(double) * n);
    double* x = (double*)malloc(sizeof(double) * S);
    if (!alpha || !F || !beta_t || !beta_next || !B_t || !B_next || !what || !x) {
      status = ORACLE_NO_MEMORY;
      free(alpha); free(F); free(beta_t); free(beta_next); free(B_t); free(B_next);
      free(what); free(x);
      continue;
    }
    dense_alpha(wq, c, lam, T, S, n, alpha, x);
    const double lz = log_sum_exp(alpha + (size_t)(n - 1) * S, S);
    for (int s = 0; s < S; ++s) beta_t[s] = 0.0;
    for (int t = n - 1; t >= 0; --t) {
      if (t < n - 1) {
        double* tmp = beta_next; beta_next = beta_t; beta_t = tmp;
        dense_beta_step(wq, c, lam, T, S, t, beta_next, beta_t, x);
      }
      double acc = 0.0;
      for (int s = 0; s < S; ++s) acc += (double)c[s] * exp(alpha[(size_t)t * S + s] + beta_t[s] - lz);
      what[t] = acc;
    }
    for (int s = 0; s < S; ++s) F[s] = 0.0;
    for (int u = 1; u < n; ++u) {
      const double* ap = alpha + (size_t)(u - 1) * S;
      const double* Fp = F + (size_t)(u - 1) * S;
      double* Fu = F + (size_t)u * S;
      for (int r = 0; r < S; ++r) {
        for (int p = 0; p < S; ++p) x[p] = ap[p] + (double)lam[(size_t)p * S + r];
        const double lse = log_sum_exp(x, S);
        double acc = 0.0;
        for (int p = 0; p < S; ++p) {
          const double pi = exp(x[p] - lse);
          const double e_prev = (double)gq[u - 1] * ((double)c[p] - what[u - 1]);
          acc += pi * (Fp[p] + e_prev);
        }
        Fu[r] = acc;
      }
    }
    for (int s = 0; s < S; ++s) { beta_t[s] = 0.0; B_t[s] = 0.0; }
    for (int u = n - 1; u >= 0; --u) {
      if (u < n - 1) {
        double* tmp = beta_next; beta_next = beta_t; beta_t = tmp;
        tmp = B_next; B_next = B_t; B_t = tmp;
        dense_beta_step(wq, c, lam, T, S, u, beta_next, beta_t, x);
        for (int r = 0; r < S; ++r) {
          double acc = 0.0;
          for (int s = 0; s < S; ++s) {
            const double rho = exp((double)lam[(size_t)r * S + s] + emission(wq[u + 1], c[s], T) +
                                   beta_next[s] - beta_t[r]);
            const double e_next = (double)gq[u + 1] * ((double)c[s] - what[u + 1]);
            acc += rho * (e_next + B_next[s]);
          }
          B_t[r] = acc;
        }
      }
      if (glq && u >= 1) { /* transitions u-1 -> u */
        for (int p = 0; p < S; ++p) {
          const double ap = alpha[(size_t)(u - 1) * S + p];
          const double past = F[(size_t)(u - 1) * S + p] + (double)gq[u - 1] * ((double)c[p] - what[u - 1]);
          for (int r = 0; r < S; ++r) {
            const double xi =
                exp(ap + (double)lam[(size_t)p * S + r] + emission(wq[u], c[r], T) + beta_t[r] - lz);
            const double future = (double)gq[u] * ((double)c[r] - what[u]) + B_t[r];
            glq[(size_t)p * S + r] += xi * (past + future);
          }
        }
      }
      double gw = 0.0;
      for (int r = 0; r < S; ++r) {
        const double gm = exp(alpha[(size_t)u * S + r] + beta_t[r] - lz);
        const double e_u = (double)gq[u] * ((double)c[r] - what[u]);
        const double psi = gm * (F[(size_t)u * S + r] + e_u + B_t[r]);
        gw += psi * (double)c[r];
        gcq[r] += (double)gq[u] * gm + (2.0 / T) * psi * ((double)wq[u] - (double)c[r]);
      }
      grad_w[(size_t)q * n + u] = (2.0 / T) * gw;
    }
    free(alpha); free(F); free(beta_t); free(beta_next); free(B_t); free(B_next);
    free(what); free(x);
  }
  for (int s = 0; s < S; ++s) grad_c[s] = 0.0;
  for (int q = 0; q < N; ++q)
    for (int s = 0; s < S; ++s) grad_c[s] += gc_seq[(size_t)q * S + s];
  if (grad_lam) {
    for (size_t i = 0; i < (size_t)S * S; ++i) grad_lam[i] = 0.0;
    for (int q = 0; q < N; ++q)
      for (size_t i = 0; i < (size_t)S * S; ++i) grad_lam[i] += gl_seq[(size_t)q * S * S + i];
  }
  free(gc_seq);
  free(gl_seq);
  return status;
}

int oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
