// fb_kernel.cuh -- fused BCJR forward-backward over the bitshift trellis (sm_100a).
//
// "BCJR-QAT: A Differentiable Relaxation of Trellis-Coded Weight Quantization",
// technical summary, "core mechanism": the soft codeword
//     w_hat_t = sum_s c(s) p_T(s_t = s | w)
// is the Boltzmann expectation of the emitted codeword under the path
// distribution at temperature T; "key technical innovations": the
// forward-backward recursion gives exact gradients through the trellis.
//
// Trellis: pred(s) = {(j << (L-k)) | (s >> k) : j < K}, K = 2^k; emission
// log-weight phi_t(s) = -(w_t - c(s))^2 / T; uniform start; free end.
//
// Group form (an exact rewrite of the forward-backward):
//   alpha_t(s) = phi_t(s) + A_t(s >> k),  A_{t+1}(g) = LSE_j alpha_t((j << (L-k)) | g)
//   beta_t(p)  = B_t(p & (S/K-1)),        B_{t-1}(h) = LSE_b [phi_t((h << k) | b) + B_t(((h << k) | b) & (S/K-1))]
// A sweep step is one K-term log-sum-exp per group of K states; only S/K
// group values move between threads.
//
// Arithmetic.  Base 2 throughout.  The emission and the running group values
// are float64 (the log-domain values of competing paths differ by tens of
// units at T = 0.005, where float32 rounding would accumulate along a path);
// exponentials and logarithms are the float32 MUFU ex2/lg2 of differences that
// are small for every term that matters.  Every step subtracts the exact
// team-wide maximum M_t of the incoming vector; the shifts are summed in
// float64 (C_t forward, D_t backward).  The backward log-sum-exp is referenced
// to the posterior itself: its terms are gamma_t(s) = 2^{y_b + r_h}, with
// r_h = A_t(h) - M_t + C_{t+1} + M'_t + D_t - log2 Z, so one exponential per
// state yields both the marginal and the backward recursion.
//
// Schedule.  One call = one launch.  A team (thread-block cluster) keeps NSEQ
// sequences in flight and alternates their steps; each step ends with a
// split cluster barrier whose arrive/wait brackets the other sequence's step,
// so the barrier latency hides behind useful work.  Global stores of a step
// (checkpoints, per-step tables, partial sums) are issued after the arrive,
// so its release never waits for them.  The forward values needed by the
// backward sweep are kept per step (C = 1) in a thread-private layout and
// fetched one step ahead with cp.async; with C > 1 only every C-th step is
// kept (float64) and each C-segment is recomputed bit-identically.
#pragma once
#include <cfloat>
#include <cmath>
#include <type_traits>

#include "bcjr_device.cuh"
#include "bcjr_internal.h"
#include "team.cuh"

namespace bcjr {

namespace fbk {

constexpr unsigned kFull = 0xffffffffu;

// Barrier schedule of one team.  With NSEQ = 2 on a cluster: after block b,
// wait for the phase of block b-1 (the previous step of the other sequence)
// and arrive for block b.  Global stores go between the two calls.
template <int CL, int NSEQ>
struct Pipe {
  bool pending = false;
  __device__ __forceinline__ void before_stores() {
    if constexpr (CL == 1) {
      __syncthreads();
    } else if constexpr (NSEQ == 1) {
      cluster_arrive();
    } else {
      if (pending) cluster_wait();
      cluster_arrive();
      pending = true;
    }
  }
  __device__ __forceinline__ void after_stores() {
    if constexpr (CL > 1 && NSEQ == 1) cluster_wait();
  }
  __device__ __forceinline__ void drain() {
    if constexpr (CL > 1 && NSEQ == 2) {
      if (pending) cluster_wait();
      pending = false;
    }
  }
};

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
  float m = -INFINITY;
  for (int i = tm.lane; i < tm.wpt; i += 32) m = fmaxf(m, maxp_buf[i]);
  return group_max(m, 32);
}
// Team-wide sum in a fixed order (every thread gets the same bits).
template <int K, int CL>
__device__ __forceinline__ double team_sum(const Team<K, CL>& tm, float* red, float v) {
  v = group_sum(v, tm.width);
  if (tm.TS <= 32) return static_cast<double>(v);
  if (tm.lane == 0) {
#pragma unroll
    for (int r = 0; r < CL; ++r) team_store<CL>(red, r, tm.warp_in_team, v);
  }
  team_sync<CL>();
  double s = 0.0;
  for (int i = 0; i < tm.wpt; ++i) s += static_cast<double>(red[i]);
  team_sync<CL>();
  return s;
}

}  // namespace fbk

template <int K, int CL, bool ADJ, int NSEQ, int NTB>
__global__ void __launch_bounds__(NTB, 1) fb_kernel(const FBParams p) {
  using TL = Tile<K>;
  constexpr int U = TL::U, JT = TL::JT, BT = TL::BT, NV = U * JT;
  const int L = p.L, k = p.k, n = p.n, C = p.C;
  const bool alias = (C == 1);
  const int S = 1 << L;
  const int TS = S / kStatesPerThread;
  const int NT = static_cast<int>(blockDim.x);
  const int tpc = (CL == 1 && TS < NT) ? NT / TS : 1;
  const int team_in_cta = (tpc > 1) ? static_cast<int>(threadIdx.x) / TS : 0;
  Team<K, CL> tm;
  tm.init(L, k, team_in_cta * TS);
  const int slot = (CL > 1) ? static_cast<int>(blockIdx.x) / CL : static_cast<int>(blockIdx.x) * tpc + team_in_cta;
  const int GL = tm.GL;
  // The K (k <= 2: all U*K) outputs of a forward step land in consecutive slots of one CTA.
  const bool contig = (K <= 4) && (L >= 3 * k);

  extern __shared__ __align__(16) unsigned char smem_raw[];
  const FBSmem lay = fb_smem_layout(GL, NT, NV, NSEQ, ADJ, alias, tpc);
  unsigned char* team_base = smem_raw + static_cast<size_t>(team_in_cta) * lay.per_team;
  float* red = reinterpret_cast<float*>(smem_raw + lay.red);

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

  // Every CTA of the cluster must be running before any of them writes into
  // another's shared memory.
  if constexpr (CL > 1) cluster_sync_all();

  const double sc64 = p.sc64;
  const int tvo = tm.tt * NV;  // this thread's offset in a thread-private row
  const int nsl = p.num_slots;
  const int iters = (p.N + nsl * NSEQ - 1) / (nsl * NSEQ);

  // Per-sequence state (identical in every thread of the team).
  struct Seq {
    int seq;
    bool act;
    float M;      // team max of the incoming vector, subtracted on read
    float Mpend;  // this step's max when the team fits in a warp
    double acc;   // forward: C_t;  backward: D_t - log2 Z
    double logZ;
    float Dc;     // backward call: E[sum_t g_t (c(s_t) - w_hat_t)]
  };

  for (int it = 0; it < iters; ++it) {
    Seq sq[NSEQ];
#pragma unroll
    for (int x = 0; x < NSEQ; ++x) {
      const int s = slot + (it * NSEQ + x) * nsl;
      sq[x].act = s < p.N;
      sq[x].seq = sq[x].act ? s : p.N - 1;
      sq[x].M = 0.f;
      sq[x].Mpend = 0.f;
      sq[x].acc = 0.0;
      sq[x].logZ = 0.0;
      sq[x].Dc = 0.f;
    }
    fbk::Pipe<CL, NSEQ> pipe;

    // ---------------- forward block: A_t -> raw A_{t+1} ----------------
    auto alpha_block = [&](auto xc, int t) {
      constexpr int X = decltype(xc)::value;
      Seq& c = sq[X];
      unsigned char* sb = team_base + static_cast<size_t>(X) * lay.per_seq;
      double* exA_r = reinterpret_cast<double*>(sb + lay.exA) + (t & 1) * GL;
      double* exA_w = reinterpret_cast<double*>(sb + lay.exA) + ((t + 1) & 1) * GL;
      float* exF_r = reinterpret_cast<float*>(sb + lay.exF) + (t & 1) * GL;
      float* exF_w = reinterpret_cast<float*>(sb + lay.exF) + ((t + 1) & 1) * GL;
      float* mp_r = reinterpret_cast<float*>(sb + lay.maxp) + (t & 1) * 128;
      float* mp_w = reinterpret_cast<float*>(sb + lay.maxp) + ((t + 1) & 1) * 128;
      const size_t lane_id = static_cast<size_t>(slot) * NSEQ + X;
      const float* wrow = p.w + static_cast<size_t>(c.seq) * n;
      if (t > 0) {
        const float Mn = fbk::collect_max(tm, mp_r, c.Mpend);
        c.acc += static_cast<double>(c.M);
        c.M = Mn;
      }
      const double Mt = static_cast<double>(c.M);
      const float wt = __ldg(wrow + t);
      float gt = 0.f, gw = 0.f;
      if constexpr (ADJ) {
        gt = __ldg(p.g + static_cast<size_t>(c.seq) * n + t);
        gw = gt * __ldg(p.what_in + static_cast<size_t>(c.seq) * n + t);
      }
      if (t + 1 < n && tm.lane == 0) {
        asm volatile("prefetch.global.L1 [%0];" ::"l"(wrow + t + 1));
        if constexpr (ADJ) {
          asm volatile("prefetch.global.L1 [%0];" ::"l"(p.g + static_cast<size_t>(c.seq) * n + t + 1));
          asm volatile("prefetch.global.L1 [%0];" ::"l"(p.what_in + static_cast<size_t>(c.seq) * n + t + 1));
        }
      }
      const double wt64 = static_cast<double>(wt);
      double a[U][JT];
      float f[U][JT];
#pragma unroll
      for (int u = 0; u < U; ++u)
#pragma unroll
        for (int jj = 0; jj < JT; ++jj) {
          a[u][jj] = (t == 0) ? 0.0 : exA_r[tm.a_read_off(u, jj)] - Mt;
          if constexpr (ADJ) f[u][jj] = (t == 0) ? 0.f : exF_r[tm.a_read_off(u, jj)];
        }
      float lmax = -INFINITY;
      double outs[U][BT];
      float fos[U][BT];
#pragma unroll
      for (int u = 0; u < U; ++u) {
#pragma unroll
        for (int bb = 0; bb < BT; ++bb) {
          double xv[JT];
          float m32 = -INFINITY;
#pragma unroll
          for (int jj = 0; jj < JT; ++jj) {
            const double d = wt64 - static_cast<double>(cb[u][jj][bb]);
            xv[jj] = fma(-sc64 * d, d, a[u][jj]);
            m32 = fmaxf(m32, static_cast<float>(xv[jj]));
          }
          if constexpr (K >= 8) {
#pragma unroll
            for (int o = TL::NBT; o < TL::TPU; o <<= 1) m32 = fmaxf(m32, __shfl_xor_sync(fbk::kFull, m32, o));
          }
          // reference point: the largest term rounded to float (any nearby value is exact for the LSE)
          const double m = static_cast<double>(m32);
          float s = 0.f, num = 0.f;
#pragma unroll
          for (int jj = 0; jj < JT; ++jj) {
            const float e = ex2f(static_cast<float>(xv[jj] - m));
            s += e;
            if constexpr (ADJ) num = fmaf(e, f[u][jj] + fmaf(gt, cb[u][jj][bb], -gw), num);
          }
          if constexpr (K >= 8) {
#pragma unroll
            for (int o = TL::NBT; o < TL::TPU; o <<= 1) {
              s += __shfl_xor_sync(fbk::kFull, s, o);
              if constexpr (ADJ) num += __shfl_xor_sync(fbk::kFull, num, o);
            }
          }
          outs[u][bb] = m + static_cast<double>(lg2f(s));
          if constexpr (ADJ) fos[u][bb] = num * rcpf(s);
          lmax = fmaxf(lmax, static_cast<float>(outs[u][bb]));
        }
      }
      if (tm.a_writer) {
        if (contig) {
          // k <= 2: the U*K outputs are consecutive slots of one CTA.
          uint32_t r;
          int off;
          tm.a_dest(tm.a_out_index(0, 0), r, off);
#pragma unroll
          for (int v = 0; v < U * BT; v += 2) {
            const double o0 = outs[v / BT][v % BT], o1 = outs[(v + 1) / BT][(v + 1) % BT];
            if constexpr (CL == 1) {
              *reinterpret_cast<double2*>(exA_w + off + v) = make_double2(o0, o1);
            } else {
              st_cluster_v2f64(exA_w + off + v, r, o0, o1);
            }
            if constexpr (ADJ) {
              team_store<CL>(exF_w, r, off + v, fos[v / BT][v % BT]);
              team_store<CL>(exF_w, r, off + v + 1, fos[(v + 1) / BT][(v + 1) % BT]);
            }
          }
        } else {
#pragma unroll
          for (int u = 0; u < U; ++u)
#pragma unroll
            for (int bb = 0; bb < BT; ++bb) {
              uint32_t r;
              int off;
              tm.a_dest(tm.a_out_index(u, bb), r, off);
              team_store_f64<CL>(exA_w, r, off, outs[u][bb]);
              if constexpr (ADJ) team_store<CL>(exF_w, r, off, fos[u][bb]);
            }
        }
      } else {
        lmax = -INFINITY;
      }
      c.Mpend = fbk::publish_max(tm, mp_w, lmax);
      pipe.before_stores();
      // ---- this step's global stores (outside the barrier's release) ----
      if (C == 1) {
        float* row = p.ck + lane_id * p.ck_stride + static_cast<size_t>(t) * p.row + tvo;
        float* rowF = ADJ ? p.ckF + lane_id * p.ck_stride + static_cast<size_t>(t) * p.row + tvo : nullptr;
#pragma unroll
        for (int v = 0; v < NV; v += 4) {
          *reinterpret_cast<float4*>(row + v) = make_float4(
              static_cast<float>(a[v / JT][v % JT]), static_cast<float>(a[(v + 1) / JT][(v + 1) % JT]),
              static_cast<float>(a[(v + 2) / JT][(v + 2) % JT]), static_cast<float>(a[(v + 3) / JT][(v + 3) % JT]));
          if constexpr (ADJ)
            *reinterpret_cast<float4*>(rowF + v) =
                make_float4(f[v / JT][v % JT], f[(v + 1) / JT][(v + 1) % JT], f[(v + 2) / JT][(v + 2) % JT],
                            f[(v + 3) / JT][(v + 3) % JT]);
        }
      } else if (t % C == 0) {
        double* row = p.ck64 + lane_id * p.ck64_stride + static_cast<size_t>(t / C) * p.row + tvo;
        float* rowF = ADJ ? p.ckF64 + lane_id * p.ck64_stride + static_cast<size_t>(t / C) * p.row + tvo : nullptr;
#pragma unroll
        for (int v = 0; v < NV; ++v) {
          row[v] = a[v / JT][v % JT];
          if constexpr (ADJ) rowF[v] = f[v / JT][v % JT];
        }
      }
      if (tm.tt == 0) {
        p.Mtab[lane_id * p.tab_stride + t] = c.M;
        p.Ctab[lane_id * p.tab_stride + t] = c.acc + Mt;
      }
      pipe.after_stores();
    };

    for (int t = 0; t < n; ++t) {
      alpha_block(std::integral_constant<int, 0>{}, t);
      if constexpr (NSEQ == 2) alpha_block(std::integral_constant<int, 1>{}, t);
    }
    pipe.drain();

    // log2 Z = C_n + log2 sum_g 2^{A_n(g)};  D = E[sum_t g_t (c(s_t) - w_hat_t)] (backward call).
    auto finish_forward = [&](auto xc) {
      constexpr int X = decltype(xc)::value;
      Seq& c = sq[X];
      unsigned char* sb = team_base + static_cast<size_t>(X) * lay.per_seq;
      const double* exA_r = reinterpret_cast<const double*>(sb + lay.exA) + (n & 1) * GL;
      const float* exF_r = reinterpret_cast<const float*>(sb + lay.exF) + (n & 1) * GL;
      const float Mn = fbk::collect_max(tm, reinterpret_cast<float*>(sb + lay.maxp) + (n & 1) * 128, c.Mpend);
      const double Cn = c.acc + static_cast<double>(c.M);
      float s1 = 0.f, s2 = 0.f;
      if (tm.b_writer) {  // one reader per group value
#pragma unroll
        for (int u = 0; u < U; ++u)
#pragma unroll
          for (int jj = 0; jj < JT; ++jj) {
            const float e = ex2f(static_cast<float>(exA_r[tm.a_read_off(u, jj)] - static_cast<double>(Mn)));
            s1 += e;
            if constexpr (ADJ) s2 = fmaf(e, exF_r[tm.a_read_off(u, jj)], s2);
          }
      }
      const double S1 = fbk::team_sum(tm, red, s1);
      const double S2 = ADJ ? fbk::team_sum(tm, red + 128, s2) : 0.0;
      c.logZ = Cn + static_cast<double>(Mn) + log2(S1);
      c.Dc = ADJ ? static_cast<float>(S2 / S1) : 0.f;
      if (tm.tt == 0 && c.act) {
        if (!isfinite(c.logZ)) atomicOr(p.status, kDevNonFinite);
        if constexpr (!ADJ) {
          if (p.log_z) p.log_z[c.seq] = static_cast<float>(c.logZ * 0.69314718055994530942);
        }
      }
      c.M = 0.f;
      c.Mpend = 0.f;
      c.acc = -c.logZ;  // backward: D_t - log2 Z with D_{n-1} = 0
    };
    finish_forward(std::integral_constant<int, 0>{});
    if constexpr (NSEQ == 2) finish_forward(std::integral_constant<int, 1>{});
    team_sync<CL>();

    // ---------------- backward block: B_t -> gamma_t, raw B_{t-1} ----------------
    auto beta_block = [&](auto xc, int t) {
      constexpr int X = decltype(xc)::value;
      Seq& c = sq[X];
      unsigned char* sb = team_base + static_cast<size_t>(X) * lay.per_seq;
      const size_t lane_id = static_cast<size_t>(slot) * NSEQ + X;
      const float* wrow = p.w + static_cast<size_t>(c.seq) * n;
      const double* ctab = p.Ctab + lane_id * p.tab_stride;
      // C > 1: recompute this C-segment's forward values (one sequence in flight).
      if (C > 1 && (t == n - 1 || (t + 1) % C == 0)) {
        const int t0 = t - (t % C);
        const float* mtab = p.Mtab + lane_id * p.tab_stride;
        for (int tp = t0; tp <= t; ++tp) {
          double* exA_r = reinterpret_cast<double*>(sb + lay.exA) + (tp & 1) * GL;
          double* exA_w = reinterpret_cast<double*>(sb + lay.exA) + ((tp + 1) & 1) * GL;
          float* exF_r = reinterpret_cast<float*>(sb + lay.exF) + (tp & 1) * GL;
          float* exF_w = reinterpret_cast<float*>(sb + lay.exF) + ((tp + 1) & 1) * GL;
          const double Mtp = static_cast<double>(mtab[tp]);
          float* ring = p.ck + lane_id * p.ck_stride + static_cast<size_t>(tp - t0) * p.row + tvo;
          float* ringF = ADJ ? p.ckF + lane_id * p.ck_stride + static_cast<size_t>(tp - t0) * p.row + tvo : nullptr;
          const double* c64 = p.ck64 + lane_id * p.ck64_stride + static_cast<size_t>(t0 / C) * p.row + tvo;
          const float* cF64 = ADJ ? p.ckF64 + lane_id * p.ck64_stride + static_cast<size_t>(t0 / C) * p.row + tvo
                                  : nullptr;
          double a[U][JT];
          float f[U][JT];
#pragma unroll
          for (int u = 0; u < U; ++u)
#pragma unroll
            for (int jj = 0; jj < JT; ++jj) {
              if (tp == t0) {
                a[u][jj] = (tp == 0) ? 0.0 : c64[u * JT + jj];
                if constexpr (ADJ) f[u][jj] = (tp == 0) ? 0.f : cF64[u * JT + jj];
              } else {
                a[u][jj] = exA_r[tm.a_read_off(u, jj)] - Mtp;
                if constexpr (ADJ) f[u][jj] = exF_r[tm.a_read_off(u, jj)];
              }
              ring[u * JT + jj] = static_cast<float>(a[u][jj]);
              if constexpr (ADJ) ringF[u * JT + jj] = f[u][jj];
            }
          if (tp < t) {
            const double wt64 = static_cast<double>(__ldg(wrow + tp));
            float gt = 0.f, gw = 0.f;
            if constexpr (ADJ) {
              gt = __ldg(p.g + static_cast<size_t>(c.seq) * n + tp);
              gw = gt * __ldg(p.what_in + static_cast<size_t>(c.seq) * n + tp);
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
#pragma unroll
              for (int bb = 0; bb < BT; ++bb) {
                double xv[JT];
                float m32 = -INFINITY;
#pragma unroll
                for (int jj = 0; jj < JT; ++jj) {
                  const double d = wt64 - static_cast<double>(cb[u][jj][bb]);
                  xv[jj] = fma(-sc64 * d, d, a[u][jj]);
                  m32 = fmaxf(m32, static_cast<float>(xv[jj]));
                }
                if constexpr (K >= 8) {
#pragma unroll
                  for (int o = TL::NBT; o < TL::TPU; o <<= 1) m32 = fmaxf(m32, __shfl_xor_sync(fbk::kFull, m32, o));
                }
                const double m = static_cast<double>(m32);
                float s = 0.f, num = 0.f;
#pragma unroll
                for (int jj = 0; jj < JT; ++jj) {
                  const float e = ex2f(static_cast<float>(xv[jj] - m));
                  s += e;
                  if constexpr (ADJ) num = fmaf(e, f[u][jj] + fmaf(gt, cb[u][jj][bb], -gw), num);
                }
                if constexpr (K >= 8) {
#pragma unroll
                  for (int o = TL::NBT; o < TL::TPU; o <<= 1) {
                    s += __shfl_xor_sync(fbk::kFull, s, o);
                    if constexpr (ADJ) num += __shfl_xor_sync(fbk::kFull, num, o);
                  }
                }
                if (tm.a_writer) {
                  uint32_t r;
                  int off;
                  tm.a_dest(tm.a_out_index(u, bb), r, off);
                  team_store_f64<CL>(exA_w, r, off, m + static_cast<double>(lg2f(s)));
                  if constexpr (ADJ) team_store<CL>(exF_w, r, off, num * rcpf(s));
                }
              }
            }
          }
          team_sync<CL>();
        }
      }

      const double* exB_r = reinterpret_cast<const double*>(sb + lay.exB) + (t & 1) * GL;
      double* exB_w = reinterpret_cast<double*>(sb + lay.exB) + ((t + 1) & 1) * GL;  // (t-1) & 1
      const float* exBt_r = reinterpret_cast<const float*>(sb + lay.exBt) + (t & 1) * GL;
      float* exBt_w = reinterpret_cast<float*>(sb + lay.exBt) + ((t + 1) & 1) * GL;
      float* mp_r = reinterpret_cast<float*>(sb + lay.maxp) + (t & 1) * 128;
      float* mp_w = reinterpret_cast<float*>(sb + lay.maxp) + ((t + 1) & 1) * 128;
      float* stg_r = reinterpret_cast<float*>(smem_raw + lay.stage) + (static_cast<size_t>(X * 2 + (t & 1)) * NT + threadIdx.x) * NV;
      float* stg_w = reinterpret_cast<float*>(smem_raw + lay.stage) + (static_cast<size_t>(X * 2 + ((t + 1) & 1)) * NT + threadIdx.x) * NV;
      float* stgF_r = reinterpret_cast<float*>(smem_raw + lay.stageF) + (static_cast<size_t>(X * 2 + (t & 1)) * NT + threadIdx.x) * NV;
      float* stgF_w = reinterpret_cast<float*>(smem_raw + lay.stageF) + (static_cast<size_t>(X * 2 + ((t + 1) & 1)) * NT + threadIdx.x) * NV;
      if (t < n - 1) {
        const float Mn = fbk::collect_max(tm, mp_r, c.Mpend);
        c.acc += static_cast<double>(c.M);
        c.M = Mn;
      }
      const double Mbt = static_cast<double>(c.M);
      // forward values A_t(h) - M_t (and F_t(h)) at the thread's groups h
      float ra[NV], fa[NV];
      if (C == 1) {
        if constexpr (NSEQ == 2) {
          cp_async_wait<1>();
        } else {
          cp_async_wait<0>();
        }
#pragma unroll
        for (int v = 0; v < NV; v += 4) {
          const float4 q4 = *reinterpret_cast<const float4*>(stg_r + v);
          ra[v] = q4.x;
          ra[v + 1] = q4.y;
          ra[v + 2] = q4.z;
          ra[v + 3] = q4.w;
          if constexpr (ADJ) {
            const float4 f4 = *reinterpret_cast<const float4*>(stgF_r + v);
            fa[v] = f4.x;
            fa[v + 1] = f4.y;
            fa[v + 2] = f4.z;
            fa[v + 3] = f4.w;
          }
        }
        if (t >= 1) {
          const float* src = p.ck + lane_id * p.ck_stride + static_cast<size_t>(t - 1) * p.row + tvo;
          const float* srcF = ADJ ? p.ckF + lane_id * p.ck_stride + static_cast<size_t>(t - 1) * p.row + tvo : nullptr;
#pragma unroll
          for (int v = 0; v < NV; v += 4) {
            cp_async16(stg_w + v, src + v);
            if constexpr (ADJ) cp_async16(stgF_w + v, srcF + v);
          }
        }
        cp_async_commit();
      } else {
        const int t0 = t - (t % C);
        const float* ring = p.ck + lane_id * p.ck_stride + static_cast<size_t>(t - t0) * p.row + tvo;
        const float* ringF = ADJ ? p.ckF + lane_id * p.ck_stride + static_cast<size_t>(t - t0) * p.row + tvo : nullptr;
#pragma unroll
        for (int v = 0; v < NV; ++v) {
          ra[v] = ring[v];
          if constexpr (ADJ) fa[v] = ringF[v];
        }
      }
      const double kap = ctab[t] + Mbt + c.acc;  // C_{t+1} + M'_t + D_t - log2 Z
      const float wt = __ldg(wrow + t);
      const double wt64 = static_cast<double>(wt);
      float gt = 0.f, gw = 0.f;
      if constexpr (ADJ) {
        gt = __ldg(p.g + static_cast<size_t>(c.seq) * n + t);
        gw = gt * __ldg(p.what_in + static_cast<size_t>(c.seq) * n + t);
      }
      if (t >= 1 && tm.lane == 0) {
        asm volatile("prefetch.global.L1 [%0];" ::"l"(wrow + t - 1));
        asm volatile("prefetch.global.L1 [%0];" ::"l"(ctab + t - 1));
        if constexpr (ADJ) {
          asm volatile("prefetch.global.L1 [%0];" ::"l"(p.g + static_cast<size_t>(c.seq) * n + t - 1));
          asm volatile("prefetch.global.L1 [%0];" ::"l"(p.what_in + static_cast<size_t>(c.seq) * n + t - 1));
        }
      }
      // incoming B_t (normalised) at the thread's successor groups (q << k) | b
      double bv[U][BT];
      float btl[U][BT];
#pragma unroll
      for (int u = 0; u < U; ++u)
#pragma unroll
        for (int bb = 0; bb < BT; ++bb) {
          bv[u][bb] = (t == n - 1) ? 0.0 : exB_r[tm.b_read_off(u, bb)] - Mbt;
          if constexpr (ADJ) btl[u][bb] = (t == n - 1) ? 0.f : exBt_r[tm.b_read_off(u, bb)];
        }
      const float tw = p.two_over_T * wt;
      float acc0 = 0.f, acc1 = 0.f;
      float lmax = -INFINITY;
      float* mrow = (!ADJ && p.marginals && c.act)
                        ? p.marginals + (static_cast<size_t>(c.seq) * n + t) * static_cast<size_t>(S)
                        : nullptr;
#pragma unroll
      for (int u = 0; u < U; ++u) {
#pragma unroll
        for (int jj = 0; jj < JT; ++jj) {
          const double r = static_cast<double>(ra[u * JT + jj]) + kap;
          float s = 0.f, bnum = 0.f;
          const float fbase = ADJ ? fa[u * JT + jj] - c.Dc : 0.f;
#pragma unroll
          for (int bb = 0; bb < BT; ++bb) {
            const float cv = cb[u][jj][bb];
            const double d = wt64 - static_cast<double>(cv);
            const float gam = ex2f(static_cast<float>(fma(-sc64 * d, d, bv[u][bb]) + r));  // gamma_t(s)
            s += gam;
            if constexpr (!ADJ) {
              acc0 = fmaf(gam, cv, acc0);
              acc1 += gam;
              if (mrow) mrow[tm.state(u, jj, bb)] = gam;
            } else {
              const float eps = fmaf(gt, cv, -gw) + btl[u][bb];
              bnum = fmaf(gam, eps, bnum);
              const float psi = gam * (fbase + eps);
              acc0 = fmaf(psi, cv, acc0);
              gc[u][jj][bb] += c.act ? fmaf(gt, gam, psi * fmaf(-p.two_over_T, cv, tw)) : 0.f;
            }
          }
          if constexpr (K >= 8) {
#pragma unroll
            for (int o = 1; o < TL::NBT; o <<= 1) {
              s += __shfl_xor_sync(fbk::kFull, s, o);
              if constexpr (ADJ) bnum += __shfl_xor_sync(fbk::kFull, bnum, o);
            }
          }
          if (t >= 1 && tm.b_writer) {
            const double out = (s > 0.f) ? static_cast<double>(lg2f(s)) - r : -INFINITY;
            uint32_t rk;
            int off;
            tm.b_dest(tm.b_out_index(u, jj), rk, off);
            team_store_f64<CL>(exB_w, rk, off, out);
            if constexpr (ADJ) team_store<CL>(exBt_w, rk, off, (s > 0.f) ? bnum * rcpf(s) : 0.f);
            lmax = fmaxf(lmax, static_cast<float>(out));
          }
        }
      }
      const float v0 = group_sum(acc0, tm.width);
      const float v1 = ADJ ? 0.f : group_sum(acc1, tm.width);
      if (t >= 1) c.Mpend = fbk::publish_max(tm, mp_w, lmax);
      pipe.before_stores();
      if ((tm.lane & (tm.width - 1)) == 0) {
        float* pr = p.part + lane_id * p.part_stride + static_cast<size_t>(t) * 2 * tm.wpt;
        pr[tm.warp_in_team] = v0;
        if constexpr (!ADJ) pr[tm.wpt + tm.warp_in_team] = v1;
      }
      pipe.after_stores();
    };

    // stage the forward values of step n-1 before the backward pipeline starts
    if (C == 1) {
#pragma unroll
      for (int x = 0; x < NSEQ; ++x) {
        const size_t lane_id = static_cast<size_t>(slot) * NSEQ + x;
        float* stg = reinterpret_cast<float*>(smem_raw + lay.stage) +
                     (static_cast<size_t>(x * 2 + ((n - 1) & 1)) * NT + threadIdx.x) * NV;
        float* stgF = reinterpret_cast<float*>(smem_raw + lay.stageF) +
                      (static_cast<size_t>(x * 2 + ((n - 1) & 1)) * NT + threadIdx.x) * NV;
        const float* src = p.ck + lane_id * p.ck_stride + static_cast<size_t>(n - 1) * p.row + tvo;
        const float* srcF = ADJ ? p.ckF + lane_id * p.ck_stride + static_cast<size_t>(n - 1) * p.row + tvo : nullptr;
#pragma unroll
        for (int v = 0; v < NV; v += 4) {
          cp_async16(stg + v, src + v);
          if constexpr (ADJ) cp_async16(stgF + v, srcF + v);
        }
        cp_async_commit();
      }
    }
    for (int t = n - 1; t >= 0; --t) {
      beta_block(std::integral_constant<int, 0>{}, t);
      if constexpr (NSEQ == 2) beta_block(std::integral_constant<int, 1>{}, t);
    }
    pipe.drain();
    team_sync<CL>();
    // Per-step outputs from the per-warp partial sums (fixed order: deterministic).
#pragma unroll
    for (int x = 0; x < NSEQ; ++x) {
      if (!sq[x].act) continue;
      const size_t lane_id = static_cast<size_t>(slot) * NSEQ + x;
      for (int t = tm.tt; t < n; t += tm.TS) {
        const float* pr = p.part + lane_id * p.part_stride + static_cast<size_t>(t) * 2 * tm.wpt;
        float v0 = 0.f, v1 = 0.f;
        for (int i = 0; i < tm.wpt; ++i) {
          v0 += pr[i];
          if constexpr (!ADJ) v1 += pr[tm.wpt + i];
        }
        if constexpr (!ADJ) {
          p.w_hat[static_cast<size_t>(sq[x].seq) * n + t] = v0 / v1;
        } else {
          p.grad_w[static_cast<size_t>(sq[x].seq) * n + t] = p.two_over_T * v0;
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

}  // namespace bcjr
