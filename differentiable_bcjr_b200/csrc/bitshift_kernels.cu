// bitshift_kernels.cu -- BCJR forward-backward over the bitshift trellis on sm_100a.
//
// "BCJR-QAT: A Differentiable Relaxation of Trellis-Coded Weight Quantization",
// technical summary, "core mechanism": the soft codeword
//     w_hat_t = sum_s c(s) p_T(s_t = s | w)
// is the Boltzmann expectation of the emitted codeword under the path
// distribution at temperature T; "key technical innovations": the forward-
// backward recursion gives exact gradients through the trellis, and the
// pages' own kernel fuses gather, log-sum-exp and add into one launch.
//
// Trellis (bitshift): pred(s) = {(j << (L-k)) | (s >> k) : j < K}, K = 2^k.
// Emission log-weight phi_t(s) = -(w_t - c(s))^2 / T; uniform start; free end.
//
// Group form used here (exact rewrite of the forward-backward):
//   alpha_t(s) = phi_t(s) + A_t(s >> k),   A_{t+1}(g) = LSE_j alpha_t((j << (L-k)) | g)
//   beta_t(p)  = B_t(p & (S/K - 1)),       B_{t-1}(h) = LSE_b [phi_t((h << k) | b) + B_t(((h << k) | b) & (S/K - 1))]
// so a sweep step is one K-term log-sum-exp per group of K states, and only
// the S/K group values travel between threads.  Everything is computed in
// base 2 (phi scaled by log2 e); every step subtracts the exact team-wide
// maximum of the incoming group vector and the shift is carried in float64.
//
// One launch does a whole call: the forward sweep (storing the raw group
// vector every C steps), then the backward sweep (recomputing the missing
// steps of each C-segment), then the per-step reductions of the outputs.
#include <cfloat>
#include <cmath>

#include "bcjr_device.cuh"
#include "bcjr_internal.h"

namespace bcjr {

namespace {

constexpr float kNegInf = -INFINITY;
constexpr unsigned kFull = 0xffffffffu;

// Per-thread state shared by the sweeps of one launch.
template <int K, int CL>
struct Team {
  using TL = Tile<K>;
  int L, k, S, G, Q, TS, GL, Qc;
  int tt, lane, width, wpt, warp_in_team;
  uint32_t rank;
  int q0, j0, b0, qloc0;
  bool a_writer, b_writer;

  __device__ void init(int L_, int k_, int team_in_cta_threads_offset) {
    L = L_;
    k = k_;
    S = 1 << L;
    G = S >> k;
    Q = S >> (2 * k);
    TS = S / kStatesPerThread;
    GL = G / CL;
    Qc = Q / CL;
    lane = threadIdx.x & 31;
    if constexpr (CL > 1) {
      rank = cluster_rank();
      tt = static_cast<int>(rank) * blockDim.x + threadIdx.x;
    } else {
      rank = 0;
      tt = threadIdx.x - team_in_cta_threads_offset;
    }
    width = TS < 32 ? TS : 32;
    wpt = TS < 32 ? 1 : TS / 32;
    warp_in_team = TS < 32 ? 0 : (tt >> 5);
    if constexpr (K <= 4) {
      q0 = tt * TL::U;
      j0 = 0;
      b0 = 0;
    } else {
      q0 = tt / TL::TPU;
      const int tile = tt % TL::TPU;
      j0 = 4 * (tile / TL::NBT);
      b0 = 4 * (tile % TL::NBT);
    }
    qloc0 = q0 - static_cast<int>(rank) * Qc;
    a_writer = (j0 == 0);
    b_writer = (b0 == 0);
  }
  __device__ __forceinline__ int state(int u, int jj, int bb) const {
    return ((j0 + jj) << (L - k)) | ((q0 + u) << k) | (b0 + bb);
  }
  // Forward-sweep layout: value index i lives with the unit that reads it.
  __device__ __forceinline__ int a_read_off(int u, int jj) const { return (j0 + jj) * Qc + qloc0 + u; }
  __device__ __forceinline__ void a_dest(int g, uint32_t& r, int& off) const {
    const int qq = g & (Q - 1), jj = g >> (L - 2 * k);
    r = static_cast<uint32_t>(qq / Qc);
    off = jj * Qc + (qq - static_cast<int>(r) * Qc);
  }
  // Backward-sweep layout: contiguous blocks of G/CL values per CTA.
  __device__ __forceinline__ int b_read_off(int u, int bb) const { return (qloc0 + u) * K + b0 + bb; }
  __device__ __forceinline__ void b_dest(int h, uint32_t& r, int& off) const {
    r = static_cast<uint32_t>(h / GL);
    off = h - static_cast<int>(r) * GL;
  }
  // Output index of the forward step (group of successors) and of the backward step.
  __device__ __forceinline__ int a_out_index(int u, int bb) const { return ((q0 + u) << k) | (b0 + bb); }
  __device__ __forceinline__ int b_out_index(int u, int jj) const {
    return ((j0 + jj) << (L - 2 * k)) | (q0 + u);
  }
};

// Team-wide maximum of one value per thread, published through shared memory
// of every CTA of the team; read back after the next team barrier.
template <int K, int CL>
__device__ __forceinline__ float publish_max(const Team<K, CL>& tm, float* maxp_buf, float v) {
  const float wm = group_max(v, tm.width);
  if (tm.TS > 32 && tm.lane == 0) {
#pragma unroll
    for (int r = 0; r < CL; ++r) team_store<CL>(maxp_buf, r, tm.warp_in_team, wm);
  }
  return wm;
}
template <int K, int CL>
__device__ __forceinline__ float collect_max(const Team<K, CL>& tm, const float* maxp_buf, float wm) {
  if (tm.TS <= 32) return wm;
  float m = kNegInf;
  for (int i = tm.lane; i < tm.wpt; i += 32) m = fmaxf(m, maxp_buf[i]);
  return group_max(m, 32);
}

// Team-wide sum (fixed order, so every thread gets the same bits).
template <int K, int CL>
__device__ __forceinline__ float team_sum(const Team<K, CL>& tm, float* red, float v) {
  v = group_sum(v, tm.width);
  if (tm.TS <= 32) return v;
  if (tm.lane == 0) {
#pragma unroll
    for (int r = 0; r < CL; ++r) team_store<CL>(red, r, tm.warp_in_team, v);
  }
  team_sync<CL>();
  float s = 0.f;
  for (int i = 0; i < tm.wpt; ++i) s += red[i];
  team_sync<CL>();
  return s;
}

// One forward step for the thread's states: inputs a[u][jj] = normalised
// group values A_t of the predecessor groups (f: adjoint accumulators),
// outputs the raw A_{t+1} of the thread's output groups (fo: accumulators).
//   adjoint accumulator  F_{t+1}(g) = sum_j pi_j (F_t(p_j >> k) + g_t (c(p_j) - w_hat_t)),
//   pi_j = the forward log-sum-exp's own softmax weights.
template <int K, bool ADJ>
__device__ __forceinline__ void forward_step(const float (&cb)[Tile<K>::U][Tile<K>::JT][Tile<K>::BT],
                                             float wt, float sc, float gt, float gw,
                                             const float (&a)[Tile<K>::U][Tile<K>::JT],
                                             const float (&f)[Tile<K>::U][Tile<K>::JT],
                                             float (&out)[Tile<K>::U][Tile<K>::BT],
                                             float (&fo)[Tile<K>::U][Tile<K>::BT]) {
  using TL = Tile<K>;
#pragma unroll
  for (int u = 0; u < TL::U; ++u) {
#pragma unroll
    for (int bb = 0; bb < TL::BT; ++bb) {
      float x[TL::JT];
      float m = kNegInf;
#pragma unroll
      for (int jj = 0; jj < TL::JT; ++jj) {
        const float d = wt - cb[u][jj][bb];
        x[jj] = fmaf(-sc * d, d, a[u][jj]);
        m = fmaxf(m, x[jj]);
      }
      if constexpr (K >= 8) {
#pragma unroll
        for (int o = TL::NBT; o < TL::TPU; o <<= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, o));
      }
      float s = 0.f, num = 0.f;
#pragma unroll
      for (int jj = 0; jj < TL::JT; ++jj) {
        const float e = ex2f(x[jj] - m);
        s += e;
        if constexpr (ADJ) num = fmaf(e, f[u][jj] + fmaf(gt, cb[u][jj][bb], -gw), num);
      }
      if constexpr (K >= 8) {
#pragma unroll
        for (int o = TL::NBT; o < TL::TPU; o <<= 1) {
          s += __shfl_xor_sync(kFull, s, o);
          if constexpr (ADJ) num += __shfl_xor_sync(kFull, num, o);
        }
      }
      out[u][bb] = m + lg2f(s);
      if constexpr (ADJ) fo[u][bb] = num * rcpf(s);
    }
  }
}

template <bool ADJ>
__host__ __device__ constexpr size_t fb_smem_floats_per_team(int GL) {
  return static_cast<size_t>(ADJ ? 8 : 4) * GL + 2 * 128 + 4 * 128;
}

}  // namespace

template <int K, int CL, bool ADJ, int NTB>
__global__ void __launch_bounds__(NTB, 1) fb_kernel(const FBParams p) {
  using TL = Tile<K>;
  constexpr int U = TL::U, JT = TL::JT, BT = TL::BT;
  const int L = p.L, k = p.k, n = p.n;
  const int S = 1 << L;
  const int TS = S / kStatesPerThread;
  const int tpc = (CL == 1 && TS < static_cast<int>(blockDim.x)) ? static_cast<int>(blockDim.x) / TS : 1;
  const int team_in_cta = (tpc > 1) ? static_cast<int>(threadIdx.x) / TS : 0;
  Team<K, CL> tm;
  tm.init(L, k, team_in_cta * TS);
  const int slot = (CL > 1) ? static_cast<int>(blockIdx.x) / CL : static_cast<int>(blockIdx.x) * tpc + team_in_cta;
  const int G = tm.G, GL = tm.GL;

  extern __shared__ __align__(16) float smem[];
  float* base = smem + team_in_cta * fb_smem_floats_per_team<ADJ>(GL);
  float* bufA = base;
  float* bufF = bufA + 2 * GL;
  float* bufB = bufA + (ADJ ? 4 : 2) * GL;
  float* bufBt = bufB + 2 * GL;
  float* maxp = bufA + (ADJ ? 8 : 4) * GL;
  float* red = maxp + 2 * 128;

  float cb[U][JT][BT];
#pragma unroll
  for (int u = 0; u < U; ++u)
#pragma unroll
    for (int jj = 0; jj < JT; ++jj)
#pragma unroll
      for (int bb = 0; bb < BT; ++bb) cb[u][jj][bb] = __ldg(p.codebook + tm.state(u, jj, bb));

  float gc[U][JT][BT];
  if constexpr (ADJ) {
#pragma unroll
    for (int u = 0; u < U; ++u)
#pragma unroll
      for (int jj = 0; jj < JT; ++jj)
#pragma unroll
        for (int bb = 0; bb < BT; ++bb) gc[u][jj][bb] = 0.f;
  }

  float* ckpt = p.ckpt + static_cast<size_t>(slot) * p.ckpt_stride;
  float* ckptF = ADJ ? p.ckptF + static_cast<size_t>(slot) * p.ckpt_stride : nullptr;
  float* ring = p.C > 1 ? p.ring + static_cast<size_t>(slot) * p.ring_stride : nullptr;
  float* ringF = (ADJ && p.C > 1) ? p.ringF + static_cast<size_t>(slot) * p.ring_stride : nullptr;
  float* Mst = p.Mst + static_cast<size_t>(slot) * p.mc_stride;
  double* Cst = p.Cst + static_cast<size_t>(slot) * p.mc_stride;
  float* part = p.part + static_cast<size_t>(slot) * p.part_stride;
  const int C = p.C;
  const float sc = p.sc;

  const int iters = (p.N + p.num_slots - 1) / p.num_slots;
  for (int it = 0; it < iters; ++it) {
    const int seq_raw = slot + it * p.num_slots;
    const bool active = seq_raw < p.N;
    const int seq = active ? seq_raw : p.N - 1;
    const float* wseq = p.w + static_cast<size_t>(seq) * n;
    const float* gseq = ADJ ? p.g + static_cast<size_t>(seq) * n : nullptr;
    const float* hseq = ADJ ? p.what_in + static_cast<size_t>(seq) * n : nullptr;

    // ------------------------------------------------------------------
    // Forward sweep: t = 0 .. n-1 produces raw A_{t+1}; A_0 = 0.
    // ------------------------------------------------------------------
    float Mt = 0.f;   // max of raw A_t (team-wide); subtracted on read
    double Ct = 0.0;  // A_t(true) = raw A_t + C_t  (log2 units)
    float out[U][BT], fo[U][BT];
    for (int t = 0; t < n; ++t) {
      const float wt = __ldg(wseq + t);
      float gt = 0.f, gw = 0.f;
      if constexpr (ADJ) {
        gt = __ldg(gseq + t);
        gw = gt * __ldg(hseq + t);
      }
      float a[U][JT], f[U][JT];
      const float* rA = bufA + (t & 1) * GL;
      const float* rF = bufF + (t & 1) * GL;
#pragma unroll
      for (int u = 0; u < U; ++u)
#pragma unroll
        for (int jj = 0; jj < JT; ++jj) {
          a[u][jj] = (t == 0) ? 0.f : rA[tm.a_read_off(u, jj)] - Mt;
          if constexpr (ADJ) f[u][jj] = (t == 0) ? 0.f : rF[tm.a_read_off(u, jj)];
        }
      forward_step<K, ADJ>(cb, wt, sc, gt, gw, a, f, out, fo);
      float lmax = kNegInf;
      if (tm.a_writer) {
        const bool keep = (t + 1 < n) && ((t + 1) % C == 0);
        float* crow = ckpt + static_cast<size_t>((t + 1) / C) * G;
        float* crowF = ADJ ? ckptF + static_cast<size_t>((t + 1) / C) * G : nullptr;
#pragma unroll
        for (int u = 0; u < U; ++u)
#pragma unroll
          for (int bb = 0; bb < BT; ++bb) {
            lmax = fmaxf(lmax, out[u][bb]);
            if (t + 1 < n) {
              const int gi = tm.a_out_index(u, bb);
              uint32_t r;
              int off;
              tm.a_dest(gi, r, off);
              team_store<CL>(bufA + ((t + 1) & 1) * GL, r, off, out[u][bb]);
              if constexpr (ADJ) team_store<CL>(bufF + ((t + 1) & 1) * GL, r, off, fo[u][bb]);
              if (keep) {
                crow[gi] = out[u][bb];
                if constexpr (ADJ) crowF[gi] = fo[u][bb];
              }
            }
          }
      }
      const float wm = publish_max(tm, maxp + ((t + 1) & 1) * 128, lmax);
      if (tm.tt == 0) {
        Mst[t] = Mt;
        Cst[t] = Ct;
      }
      team_sync<CL>();
      const float Mn = collect_max(tm, maxp + ((t + 1) & 1) * 128, wm);
      Ct += static_cast<double>(Mt);
      Mt = Mn;
    }
    // Now out = raw A_n (never stored), Mt = max A_n, Ct = C_n.
    // log2 Z = C_n + log2 sum_g 2^{A_n(g)};  D = E[sum_t g_t (c(s_t) - w_hat_t)].
    float s1 = 0.f, s2 = 0.f;
    if (tm.a_writer) {
#pragma unroll
      for (int u = 0; u < U; ++u)
#pragma unroll
        for (int bb = 0; bb < BT; ++bb) {
          const float e = ex2f(out[u][bb] - Mt);
          s1 += e;
          if constexpr (ADJ) s2 = fmaf(e, fo[u][bb], s2);
        }
    }
    s1 = team_sum(tm, red, s1);
    if constexpr (ADJ) s2 = team_sum(tm, red + 128, s2);
    const double log2Z = Ct + static_cast<double>(Mt) + log2(static_cast<double>(s1));
    const float Dc = ADJ ? s2 / s1 : 0.f;
    if (tm.tt == 0 && active) {
      if (!isfinite(log2Z)) atomicOr(p.status, kDevNonFinite);
      if constexpr (!ADJ) {
        if (p.log_z) p.log_z[seq] = static_cast<float>(log2Z * 0.69314718055994530942);
      }
    }

    // ------------------------------------------------------------------
    // Backward sweep: t = n-1 .. 0 consumes B_t, produces raw B_{t-1}.
    // ------------------------------------------------------------------
    float Mb = 0.f;
    double Dt = 0.0;  // B_t(true) = raw B_t + D_t
    for (int t = n - 1; t >= 0; --t) {
      // Recompute the forward group vectors of this C-segment when they were not kept.
      if (C > 1 && t >= 1 && (t == n - 1 || (t + 1) % C == 0)) {
        const int t0 = t - (t % C);
        for (int tp = t0; tp < t; ++tp) {
          const float wt = __ldg(wseq + tp);
          float gt = 0.f, gw = 0.f;
          if constexpr (ADJ) {
            gt = __ldg(gseq + tp);
            gw = gt * __ldg(hseq + tp);
          }
          const float Mtp = Mst[tp];
          float a[U][JT], f[U][JT];
          const float* crow = ckpt + static_cast<size_t>(t0 / C) * G;
          const float* crowF = ADJ ? ckptF + static_cast<size_t>(t0 / C) * G : nullptr;
#pragma unroll
          for (int u = 0; u < U; ++u)
#pragma unroll
            for (int jj = 0; jj < JT; ++jj) {
              const int gi = ((tm.j0 + jj) << (L - 2 * k)) | (tm.q0 + u);
              float av, fv = 0.f;
              if (tp == 0) {
                av = 0.f;
              } else if (tp == t0) {
                av = crow[gi] - Mtp;
                if constexpr (ADJ) fv = crowF[gi];
              } else {
                av = bufA[(tp & 1) * GL + tm.a_read_off(u, jj)] - Mtp;
                if constexpr (ADJ) fv = bufF[(tp & 1) * GL + tm.a_read_off(u, jj)];
              }
              a[u][jj] = av;
              if constexpr (ADJ) f[u][jj] = fv;
            }
          float ro[U][BT], rfo[U][BT];
          forward_step<K, ADJ>(cb, wt, sc, gt, gw, a, f, ro, rfo);
          if (tm.a_writer) {
            float* rrow = ring + static_cast<size_t>(tp + 1 - t0) * G;
            float* rrowF = ADJ ? ringF + static_cast<size_t>(tp + 1 - t0) * G : nullptr;
#pragma unroll
            for (int u = 0; u < U; ++u)
#pragma unroll
              for (int bb = 0; bb < BT; ++bb) {
                const int gi = tm.a_out_index(u, bb);
                uint32_t r;
                int off;
                tm.a_dest(gi, r, off);
                team_store<CL>(bufA + ((tp + 1) & 1) * GL, r, off, ro[u][bb]);
                rrow[gi] = ro[u][bb];
                if constexpr (ADJ) {
                  team_store<CL>(bufF + ((tp + 1) & 1) * GL, r, off, rfo[u][bb]);
                  rrowF[gi] = rfo[u][bb];
                }
              }
          }
          team_sync<CL>();
        }
      }

      const float wt = __ldg(wseq + t);
      float gt = 0.f, gw = 0.f;
      if constexpr (ADJ) {
        gt = __ldg(gseq + t);
        gw = gt * __ldg(hseq + t);
      }
      // Incoming backward group values B_t (normalised) at (q << k) | b.
      float bv[U][BT], btl[U][BT];
      const float* rB = bufB + (t & 1) * GL;
      const float* rBt = bufBt + (t & 1) * GL;
#pragma unroll
      for (int u = 0; u < U; ++u)
#pragma unroll
        for (int bb = 0; bb < BT; ++bb) {
          bv[u][bb] = (t == n - 1) ? 0.f : rB[tm.b_read_off(u, bb)] - Mb;
          if constexpr (ADJ) btl[u][bb] = (t == n - 1) ? 0.f : rBt[tm.b_read_off(u, bb)];
        }
      // Forward group values A_t at the groups h = (j << (L-2k)) | q of the thread's states.
      float ra[U][JT], fa[U][JT];
      {
        const float* row = nullptr;
        const float* rowF = nullptr;
        if (t >= 1) {
          if (C == 1 || t % C == 0) {
            row = ckpt + static_cast<size_t>(t / C) * G;
            if constexpr (ADJ) rowF = ckptF + static_cast<size_t>(t / C) * G;
          } else {
            row = ring + static_cast<size_t>(t % C) * G;
            if constexpr (ADJ) rowF = ringF + static_cast<size_t>(t % C) * G;
          }
        }
#pragma unroll
        for (int u = 0; u < U; ++u)
#pragma unroll
          for (int jj = 0; jj < JT; ++jj) {
            const int h = tm.b_out_index(u, jj);
            ra[u][jj] = (t >= 1) ? row[h] : 0.f;
            if constexpr (ADJ) fa[u][jj] = (t >= 1) ? rowF[h] : 0.f;
          }
      }
      // gamma_t(s) = 2^{y_b - m + m + A_t(h) + C_t + Mb + D_t - log2 Z}
      const float kap = static_cast<float>(static_cast<double>(Mb) + Cst[t] + Dt - log2Z);
      const float tw = p.two_over_T * wt;
      float acc0 = 0.f, acc1 = 0.f;  // forward: sum c gamma, sum gamma; backward: sum psi c
      float bo[U][JT], bto[U][JT];
      float* mrow = (!ADJ && p.marginals && active)
                        ? p.marginals + (static_cast<size_t>(seq) * n + t) * static_cast<size_t>(S)
                        : nullptr;
#pragma unroll
      for (int u = 0; u < U; ++u) {
#pragma unroll
        for (int jj = 0; jj < JT; ++jj) {
          float y[BT];
          float m = kNegInf;
#pragma unroll
          for (int bb = 0; bb < BT; ++bb) {
            const float d = wt - cb[u][jj][bb];
            y[bb] = fmaf(-sc * d, d, bv[u][bb]);
            m = fmaxf(m, y[bb]);
          }
          if constexpr (K >= 8) {
#pragma unroll
            for (int o = 1; o < TL::NBT; o <<= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, o));
          }
          float e[BT];
          float s = 0.f, ec = 0.f, bnum = 0.f;
          float eps[BT];
#pragma unroll
          for (int bb = 0; bb < BT; ++bb) {
            e[bb] = ex2f(y[bb] - m);
            s += e[bb];
            ec = fmaf(e[bb], cb[u][jj][bb], ec);
            if constexpr (ADJ) {
              eps[bb] = fmaf(gt, cb[u][jj][bb], -gw) + btl[u][bb];
              bnum = fmaf(e[bb], eps[bb], bnum);
            }
          }
          const float s_own = s;
          if constexpr (K >= 8) {
#pragma unroll
            for (int o = 1; o < TL::NBT; o <<= 1) {
              s += __shfl_xor_sync(kFull, s, o);
              if constexpr (ADJ) bnum += __shfl_xor_sync(kFull, bnum, o);
            }
          }
          bo[u][jj] = m + lg2f(s);
          if constexpr (ADJ) bto[u][jj] = bnum * rcpf(s);
          const float Gf = ex2f(m + ra[u][jj] + kap);
          if constexpr (!ADJ) {
            acc0 = fmaf(Gf, ec, acc0);
            acc1 = fmaf(Gf, s_own, acc1);
            if (mrow) {
#pragma unroll
              for (int bb = 0; bb < BT; ++bb) mrow[tm.state(u, jj, bb)] = e[bb] * Gf;
            }
          } else {
            const float base = fa[u][jj] - Dc;
#pragma unroll
            for (int bb = 0; bb < BT; ++bb) {
              const float gam = e[bb] * Gf;
              const float psi = gam * (base + eps[bb]);
              acc0 = fmaf(psi, cb[u][jj][bb], acc0);
              if (active)
                gc[u][jj][bb] += fmaf(gt, gam, psi * fmaf(-p.two_over_T, cb[u][jj][bb], tw));
            }
          }
        }
      }
      // Per-step partial sums, one pair per warp (per team when narrower).
      {
        const float v0 = group_sum(acc0, tm.width);
        const float v1 = ADJ ? 0.f : group_sum(acc1, tm.width);
        if ((tm.lane & (tm.width - 1)) == 0) {
          part[(static_cast<size_t>(t) * 2 + 0) * tm.wpt + tm.warp_in_team] = v0;
          if constexpr (!ADJ) part[(static_cast<size_t>(t) * 2 + 1) * tm.wpt + tm.warp_in_team] = v1;
        }
      }
      if (t >= 1) {
        float lmax = kNegInf;
        if (tm.b_writer) {
#pragma unroll
          for (int u = 0; u < U; ++u)
#pragma unroll
            for (int jj = 0; jj < JT; ++jj) {
              lmax = fmaxf(lmax, bo[u][jj]);
              uint32_t r;
              int off;
              tm.b_dest(tm.b_out_index(u, jj), r, off);
              team_store<CL>(bufB + ((t - 1) & 1) * GL, r, off, bo[u][jj]);
              if constexpr (ADJ) team_store<CL>(bufBt + ((t - 1) & 1) * GL, r, off, bto[u][jj]);
            }
        }
        const float wm = publish_max(tm, maxp + ((t - 1) & 1) * 128, lmax);
        team_sync<CL>();
        const float Mn = collect_max(tm, maxp + ((t - 1) & 1) * 128, wm);
        Dt += static_cast<double>(Mb);
        Mb = Mn;
      }
    }
    team_sync<CL>();
    // Per-step outputs from the partial sums (fixed order: deterministic).
    if (active) {
      for (int t = tm.tt; t < n; t += tm.TS) {
        float v0 = 0.f, v1 = 0.f;
        for (int i = 0; i < tm.wpt; ++i) {
          v0 += part[(static_cast<size_t>(t) * 2 + 0) * tm.wpt + i];
          if constexpr (!ADJ) v1 += part[(static_cast<size_t>(t) * 2 + 1) * tm.wpt + i];
        }
        if constexpr (!ADJ) {
          p.w_hat[static_cast<size_t>(seq) * n + t] = v0 / v1;
        } else {
          p.grad_w[static_cast<size_t>(seq) * n + t] = p.two_over_T * v0;
        }
      }
    }
    team_sync<CL>();
  }

  if constexpr (ADJ) {
    float* gp = p.gc_part + static_cast<size_t>(slot) * S;
#pragma unroll
    for (int u = 0; u < U; ++u)
#pragma unroll
      for (int jj = 0; jj < JT; ++jj)
#pragma unroll
        for (int bb = 0; bb < BT; ++bb) gp[tm.state(u, jj, bb)] = gc[u][jj][bb];
  }
  if constexpr (CL > 1) cluster_sync_all();  // no CTA leaves while its shared memory may be addressed
}

// ---------------------------------------------------------------------------
// Hard decode: max-sum over -(w - c)^2 in float64, each difference, square and
// sum rounded separately, ties to the lowest predecessor index and the lowest
// final state ("BCJR-QAT", technical summary: T -> 0 recovers the hard Viterbi
// output).  Backpointers (k bits, stored as bytes) go to the workspace; one
// thread of the team walks them back.
// ---------------------------------------------------------------------------
template <int K, int CL, int NTB>
__global__ void __launch_bounds__(NTB, 1) viterbi_kernel(const ViterbiParams p) {
  using TL = Tile<K>;
  constexpr int U = TL::U, JT = TL::JT, BT = TL::BT;
  const int L = p.L, k = p.k, n = p.n;
  const int S = 1 << L;
  const int TS = S / kStatesPerThread;
  const int tpc = (CL == 1 && TS < static_cast<int>(blockDim.x)) ? static_cast<int>(blockDim.x) / TS : 1;
  const int team_in_cta = (tpc > 1) ? static_cast<int>(threadIdx.x) / TS : 0;
  Team<K, CL> tm;
  tm.init(L, k, team_in_cta * TS);
  const int slot = (CL > 1) ? static_cast<int>(blockIdx.x) / CL : static_cast<int>(blockIdx.x) * tpc + team_in_cta;
  const int G = tm.G, GL = tm.GL;

  extern __shared__ __align__(16) double smemd[];
  double* base = smemd + team_in_cta * (2 * static_cast<size_t>(GL) + 2 * 128);
  double* bufV = base;                 // [2][GL]
  double* redv = bufV + 2 * GL;        // [128]
  int* reds = reinterpret_cast<int*>(redv + 128);  // [128]

  float cb[U][JT][BT];
#pragma unroll
  for (int u = 0; u < U; ++u)
#pragma unroll
    for (int jj = 0; jj < JT; ++jj)
#pragma unroll
      for (int bb = 0; bb < BT; ++bb) cb[u][jj][bb] = __ldg(p.codebook + tm.state(u, jj, bb));

  uint8_t* bp = p.bp + static_cast<size_t>(slot) * p.bp_stride;
  const int iters = (p.N + p.num_slots - 1) / p.num_slots;
  for (int it = 0; it < iters; ++it) {
    const int seq_raw = slot + it * p.num_slots;
    const bool active = seq_raw < p.N;
    const int seq = active ? seq_raw : p.N - 1;
    const float* wseq = p.w + static_cast<size_t>(seq) * n;
    double best[U][BT];
    int bj[U][BT];
    for (int t = 0; t < n; ++t) {
      const double wt = static_cast<double>(__ldg(wseq + t));
      double a[U][JT];
#pragma unroll
      for (int u = 0; u < U; ++u)
#pragma unroll
        for (int jj = 0; jj < JT; ++jj)
          a[u][jj] = (t == 0) ? 0.0 : bufV[(t & 1) * GL + tm.a_read_off(u, jj)];
#pragma unroll
      for (int u = 0; u < U; ++u)
#pragma unroll
        for (int bb = 0; bb < BT; ++bb) {
          double bv = -DBL_MAX;
          int bjj = 0;
#pragma unroll
          for (int jj = 0; jj < JT; ++jj) {
            const double d = __dsub_rn(wt, static_cast<double>(cb[u][jj][bb]));
            const double v = __dadd_rn(a[u][jj], -__dmul_rn(d, d));
            if (jj == 0 || v > bv) {
              bv = v;
              bjj = tm.j0 + jj;
            }
          }
          if constexpr (K >= 8) {
#pragma unroll
            for (int o = TL::NBT; o < TL::TPU; o <<= 1) {
              const double ov = __shfl_xor_sync(kFull, bv, o);
              const int oj = __shfl_xor_sync(kFull, bjj, o);
              if (ov > bv || (ov == bv && oj < bjj)) {
                bv = ov;
                bjj = oj;
              }
            }
          }
          best[u][bb] = bv;
          bj[u][bb] = bjj;
        }
      if (t + 1 < n && tm.a_writer) {
        uint8_t* brow = bp + static_cast<size_t>(t + 1) * G;
#pragma unroll
        for (int u = 0; u < U; ++u)
#pragma unroll
          for (int bb = 0; bb < BT; ++bb) {
            const int gi = tm.a_out_index(u, bb);
            uint32_t r;
            int off;
            tm.a_dest(gi, r, off);
            team_store_f64<CL>(bufV + ((t + 1) & 1) * GL, r, off, best[u][bb]);
            brow[gi] = static_cast<uint8_t>(bj[u][bb]);
          }
      }
      team_sync<CL>();
    }
    // End state: the largest final metric, lowest state on ties.
    double vb = -DBL_MAX;
    int sb = S;  // S marks "no candidate"; every reduction below keeps a valid state when one exists
    if (tm.a_writer) {
#pragma unroll
      for (int u = 0; u < U; ++u)
#pragma unroll
        for (int bb = 0; bb < BT; ++bb) {
          const int st = (bj[u][bb] << (L - k)) | tm.a_out_index(u, bb);
          if (sb == S || best[u][bb] > vb || (best[u][bb] == vb && st < sb)) {
            vb = best[u][bb];
            sb = st;
          }
        }
    }
    for (int o = tm.width >> 1; o > 0; o >>= 1) {
      const double ov = __shfl_xor_sync(kFull, vb, o);
      const int os = __shfl_xor_sync(kFull, sb, o);
      if (os != S && (sb == S || ov > vb || (ov == vb && os < sb))) {
        vb = ov;
        sb = os;
      }
    }
    if (tm.TS > 32) {
      if (tm.lane == 0) {
        for (int r = 0; r < CL; ++r) {
          team_store_f64<CL>(redv, r, tm.warp_in_team, vb);
          team_store_u32<CL>(reinterpret_cast<uint32_t*>(reds), r, tm.warp_in_team, static_cast<uint32_t>(sb));
        }
      }
      team_sync<CL>();
      vb = -DBL_MAX;
      sb = S;
      for (int i = 0; i < tm.wpt; ++i) {
        const double ov = redv[i];
        const int os = reds[i];
        if (os != S && (sb == S || ov > vb || (ov == vb && os < sb))) {
          vb = ov;
          sb = os;
        }
      }
    }
    // Non-finite metrics (NaN inputs) can leave no comparable candidate: keep the walk in range.
    if (sb < 0 || sb >= S) sb = 0;
    if (tm.tt == 0 && active) {
      if (!isfinite(vb)) atomicOr(p.status, kDevNonFinite);
      if (p.metric) p.metric[seq] = vb;
      int s = sb;
      int32_t* st = p.states + static_cast<size_t>(seq) * n;
      float* wh = p.w_hard ? p.w_hard + static_cast<size_t>(seq) * n : nullptr;
      for (int t = n - 1; t >= 0; --t) {
        st[t] = s;
        if (wh) wh[t] = __ldg(p.codebook + s);
        if (t >= 1) {
          const int j = bp[static_cast<size_t>(t) * G + (s >> k)];
          s = (j << (L - k)) | (s >> k);
        }
      }
    }
    team_sync<CL>();
  }
  if constexpr (CL > 1) cluster_sync_all();
}

// grad_codebook[s] (+)= sum over teams of the per-team partials, in team order.
__global__ void gradc_reduce_kernel(const float* __restrict__ part, int num_slots, int S,
                                    float* __restrict__ out, int accumulate) {
  const int s = blockIdx.x * blockDim.x + threadIdx.x;
  if (s >= S) return;
  float acc = 0.f;
  for (int i = 0; i < num_slots; ++i) acc += part[static_cast<size_t>(i) * S + s];
  out[s] = accumulate ? out[s] + acc : acc;
}

// ---------------------------------------------------------------------------
// Host side: geometry and launches.
// ---------------------------------------------------------------------------
namespace {

template <int K, int CL, bool ADJ, int NTB>
const void* fb_fn() {
  return reinterpret_cast<const void*>(&fb_kernel<K, CL, ADJ, NTB>);
}

template <bool ADJ>
const void* pick_fb(int k, int cl) {
#define BCJR_FB_CASE(KK, CC)                                  \
  if (k == KK && cl == CC) return fb_fn<(1 << KK), CC, ADJ, 1024>();
  BCJR_FB_CASE(1, 1) BCJR_FB_CASE(1, 2) BCJR_FB_CASE(1, 4)
  BCJR_FB_CASE(2, 1) BCJR_FB_CASE(2, 2) BCJR_FB_CASE(2, 4)
  BCJR_FB_CASE(3, 1) BCJR_FB_CASE(3, 2) BCJR_FB_CASE(3, 4)
  BCJR_FB_CASE(4, 1) BCJR_FB_CASE(4, 2) BCJR_FB_CASE(4, 4)
#undef BCJR_FB_CASE
  return nullptr;
}

const void* pick_viterbi(int k, int cl) {
#define BCJR_V_CASE(KK, CC) \
  if (k == KK && cl == CC) return reinterpret_cast<const void*>(&viterbi_kernel<(1 << KK), CC, 1024>);
  BCJR_V_CASE(1, 1) BCJR_V_CASE(1, 2) BCJR_V_CASE(1, 4)
  BCJR_V_CASE(2, 1) BCJR_V_CASE(2, 2) BCJR_V_CASE(2, 4)
  BCJR_V_CASE(3, 1) BCJR_V_CASE(3, 2) BCJR_V_CASE(3, 4)
  BCJR_V_CASE(4, 1) BCJR_V_CASE(4, 2) BCJR_V_CASE(4, 4)
#undef BCJR_V_CASE
  return nullptr;
}

void base_geometry(int L, TeamGeometry* g) {
  const int TS = (1 << L) / kStatesPerThread;
  g->team_threads = TS;
  if (TS > 1024) {
    g->block_threads = 1024;
    g->cluster = TS / 1024;
    g->teams_per_cta = 1;
  } else if (TS >= 32) {
    g->block_threads = TS;
    g->cluster = 1;
    g->teams_per_cta = 1;
  } else {
    g->block_threads = 32;
    g->cluster = 1;
    g->teams_per_cta = 32 / TS;
  }
  g->warps_per_team = TS < 32 ? 1 : TS / 32;
}

cudaError_t persistent_grid(const void* fn, int n_seq, TeamGeometry* g) {
  int dev0 = 0, max_smem = 0;
  cudaError_t e = cudaGetDevice(&dev0);
  if (e != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev0)) != cudaSuccess)
    return e;
  if (g->smem_bytes > static_cast<size_t>(max_smem)) return cudaErrorNotSupported;
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(g->smem_bytes));
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  int resident_teams = 0;
  if (g->cluster > 1) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(g->cluster * sms, 1, 1);
    cfg.blockDim = dim3(g->block_threads, 1, 1);
    cfg.dynamicSmemBytes = g->smem_bytes;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = g->cluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int clusters = 0;
    if ((e = cudaOccupancyMaxActiveClusters(&clusters, fn, &cfg)) != cudaSuccess) return e;
    resident_teams = clusters;
  } else {
    int per_sm = 0;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, g->block_threads, g->smem_bytes)) !=
        cudaSuccess)
      return e;
    resident_teams = per_sm * sms * g->teams_per_cta;
  }
  if (resident_teams < 1) return cudaErrorInvalidConfiguration;
  int slots = n_seq < resident_teams ? n_seq : resident_teams;
  if (slots < 1) slots = 1;
  if (g->cluster > 1) {
    g->num_slots = slots;
    g->grid_blocks = slots * g->cluster;
  } else {
    const int blocks = (slots + g->teams_per_cta - 1) / g->teams_per_cta;
    g->grid_blocks = blocks;
    g->num_slots = blocks * g->teams_per_cta;
  }
  return cudaSuccess;
}

cudaError_t launch(const void* fn, const TeamGeometry& g, void** args, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(g.grid_blocks, 1, 1);
  cfg.blockDim = dim3(g.block_threads, 1, 1);
  cfg.dynamicSmemBytes = g.smem_bytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = g.cluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = g.cluster > 1 ? 1 : 0;
  return cudaLaunchKernelExC(&cfg, fn, args);
}

}  // namespace

cudaError_t fb_geometry(int L, int k, int n_seq, bool adjoint, TeamGeometry* g) {
  base_geometry(L, g);
  const int GL = ((1 << L) >> k) / g->cluster;
  const size_t per_team = adjoint ? fb_smem_floats_per_team<true>(GL) : fb_smem_floats_per_team<false>(GL);
  g->smem_bytes = per_team * sizeof(float) * g->teams_per_cta;
  const void* fn = adjoint ? pick_fb<true>(k, g->cluster) : pick_fb<false>(k, g->cluster);
  if (!fn) return cudaErrorInvalidValue;
  return persistent_grid(fn, n_seq, g);
}

cudaError_t viterbi_geometry(int L, int k, int n_seq, TeamGeometry* g) {
  base_geometry(L, g);
  const int GL = ((1 << L) >> k) / g->cluster;
  g->smem_bytes = (2 * static_cast<size_t>(GL) + 2 * 128) * sizeof(double) * g->teams_per_cta;
  const void* fn = pick_viterbi(k, g->cluster);
  if (!fn) return cudaErrorInvalidValue;
  return persistent_grid(fn, n_seq, g);
}

cudaError_t launch_fb(const FBParams& p, const TeamGeometry& g, bool adjoint, cudaStream_t s) {
  const void* fn = adjoint ? pick_fb<true>(p.k, g.cluster) : pick_fb<false>(p.k, g.cluster);
  if (!fn) return cudaErrorInvalidValue;
  FBParams copy = p;
  void* args[] = {&copy};
  return launch(fn, g, args, s);
}

cudaError_t launch_viterbi(const ViterbiParams& p, const TeamGeometry& g, cudaStream_t s) {
  const void* fn = pick_viterbi(p.k, g.cluster);
  if (!fn) return cudaErrorInvalidValue;
  ViterbiParams copy = p;
  void* args[] = {&copy};
  return launch(fn, g, args, s);
}

cudaError_t launch_gradc_reduce(const float* gc_part, int num_slots, int S, float* grad_c, int accumulate,
                                cudaStream_t s) {
  const int threads = 256;
  gradc_reduce_kernel<<<(S + threads - 1) / threads, threads, 0, s>>>(gc_part, num_slots, S, grad_c,
                                                                        accumulate);
  return cudaGetLastError();
}

}  // namespace bcjr
