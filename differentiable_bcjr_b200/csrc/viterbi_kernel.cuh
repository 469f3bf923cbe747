// viterbi_kernel.cuh -- hard decode over the bitshift trellis (sm_100a).
//
// "BCJR-QAT: A Differentiable Relaxation of Trellis-Coded Weight Quantization",
// technical summary: the T -> 0 limit of the Boltzmann path distribution is
// the hard Viterbi code.  Max-sum over -(w_t - c(s))^2 in float64, with the
// difference, the square and the sum each rounded separately (no fused
// multiply-add), so the path metrics are those of a plain sequential max-sum;
// ties go to the lowest predecessor index j and the lowest final state.
//
// Same team layout and exchange as the forward-backward kernel: a sequence
// spans a thread-block cluster, group maxima travel with st.async into the
// reader CTA's double-buffered shared memory and are awaited on mbarriers; the
// relaxed split cluster barrier orders buffer reuse, and two sequences are in
// flight per cluster.  Backpointers (the argmax j, one byte per group and
// step, packed into one store per thread-step) go to a double-buffered
// workspace area; one thread per sequence walks them back during the forward
// steps of the next sequences, one walk step per forward step, so that the
// latency of each dependent load hides behind a step of max-sum work.
#pragma once
#include <cfloat>
#include <cmath>
#include <type_traits>

#include "bcjr_device.cuh"
#include "bcjr_internal.h"
#include "fb_kernel.cuh"  // fbk::Pipe, the split cluster barrier schedule
#include "team.cuh"

namespace bcjr {

template <int K, int CL, int NSEQ, int NTB>
__global__ void __launch_bounds__(NTB, 1) viterbi_kernel(const ViterbiParams p) {
  using TL = Tile<K>;
  constexpr int U = TL::U, JT = TL::JT, BT = TL::BT;
  constexpr int NB = U * BT;  // backpointers a writer thread produces per step (4 or 8)
  // Backpointers are packed at KB bits each (k bits for k <= 2, 4 bits for
  // k = 3, 4), so a writer thread's NB values fill one byte (k <= 2) or two.
  constexpr int KB = K <= 4 ? ilog2_constexpr(K) : 4;
  static_assert(NB * KB == 8 || NB * KB == 16, "one or two bytes per writer thread and step");
  constexpr int k = K == 2 ? 1 : K == 4 ? 2 : K == 8 ? 3 : 4;
  // A cluster team fills its cluster exactly, so the trellis size is then a constant.
  constexpr int kLc = CL > 1 ? ilog2_constexpr(kStatesPerThread * CL * NTB) : 0;
  constexpr unsigned kFullMask = 0xffffffffu;
  const int L = kLc ? kLc : p.L;
  const int n = p.n;
  const int S = 1 << L;
  const int TS = S / kStatesPerThread;
  const int NT = CL > 1 ? NTB : static_cast<int>(blockDim.x);
  const int tpc = (CL == 1 && TS < NT) ? NT / TS : 1;
  const int team_in_cta = (tpc > 1) ? static_cast<int>(threadIdx.x) / TS : 0;
  Team<K, CL> tm;
  tm.init(L, k, team_in_cta * TS);
  const int slot = (CL > 1) ? static_cast<int>(blockIdx.x) / CL : static_cast<int>(blockIdx.x) * tpc + team_in_cta;
  const int G = tm.G, GL = tm.GL;
  const size_t row_bytes = static_cast<size_t>(G) * KB / 8;  // backpointers of one step
  const bool contig = (K <= 4) && (L >= 3 * k);

  // Shared memory (doubles): per team, per sequence in flight [2][GL] group
  // maxima + 2 mbarriers; then a reduction scratch of 128 doubles + 128 ints.
  extern __shared__ __align__(16) double smemd[];
  const int per_seq = 2 * GL + 2;
  const int per_team = NSEQ * per_seq + 192;
  double* team_base = smemd + static_cast<size_t>(team_in_cta) * per_team;
  double* redv = team_base + NSEQ * per_seq;
  int* reds = reinterpret_cast<int*>(redv + 128);
  auto bufV = [&](int X, int par) { return team_base + X * per_seq + par * GL; };
  auto mbar = [&](int X, int par) { return reinterpret_cast<uint64_t*>(team_base + X * per_seq + 2 * GL) + par; };

  double cpd[U][JT][BT];  // codewords as float64 (exact)
#pragma unroll
  for (int u = 0; u < U; ++u)
#pragma unroll
    for (int jj = 0; jj < JT; ++jj)
#pragma unroll
      for (int bb = 0; bb < BT; ++bb) cpd[u][jj][bb] = static_cast<double>(__ldg(p.codebook + tm.state(u, jj, bb)));

  uint32_t ph[NSEQ];
#pragma unroll
  for (int x = 0; x < NSEQ; ++x) ph[x] = 0;
  bool timed_out = false;
  if constexpr (CL > 1) {
    if (threadIdx.x == 0) {
#pragma unroll
      for (int x = 0; x < NSEQ; ++x) {
        mbar_init(mbar(x, 0), 1);
        mbar_init(mbar(x, 1), 1);
      }
      mbar_init_fence();
    }
    cluster_sync_all();
  }
  const uint32_t xbytes = static_cast<uint32_t>(GL) * 8u;
  auto xwait = [&](int X, int par) {
    if constexpr (CL > 1) {
      if (!timed_out) timed_out = !mbar_wait(mbar(X, par), (ph[X] >> par) & 1u, p.status, kDevTimeout);
      ph[X] ^= 1u << par;
    }
  };
  auto xarm = [&](int X, int par) {
    if constexpr (CL > 1) {
      if (threadIdx.x == 0) mbar_arm(mbar(X, par), xbytes);
    }
  };

  const int nsl = p.num_slots;
  const int iters = (p.N + nsl * NSEQ - 1) / (nsl * NSEQ);
  // Backpointers of sequence slot X in iteration `it` (two buffers, by the parity of it).
  auto bp_buf = [&](int X, int it_) {
    return p.bp + ((static_cast<size_t>(slot) * NSEQ + X) * 2 + (it_ & 1)) * p.bp_stride;
  };
  // The walker of sequence slot X: lane 0 of warp X of the team.
  auto is_walker = [&](int X) { return tm.tt == 32 * X; };
  // Walk state of the previous sequence in each slot (kept by its walker).
  int wk_s[NSEQ], wk_j[NSEQ], wk_seq[NSEQ];
  bool wk_act[NSEQ];
  const uint8_t* wk_bp[NSEQ];
#pragma unroll
  for (int x = 0; x < NSEQ; ++x) {
    wk_s[x] = 0;
    wk_j[x] = 0;
    wk_seq[x] = 0;
    wk_act[x] = false;
    wk_bp[x] = nullptr;
  }
  // One walk step at time index ti (counting down from n-1); the backpointer
  // loaded here is consumed by the next step.
  auto walk_step = [&](int x, int ti) {
    if (ti < n - 1) wk_s[x] = (wk_j[x] << (L - k)) | (wk_s[x] >> k);
    p.states[static_cast<size_t>(wk_seq[x]) * n + ti] = wk_s[x];
    if (ti >= 1) {
      const int bit = (wk_s[x] >> k) * KB;
      wk_j[x] = (wk_bp[x][static_cast<size_t>(ti) * row_bytes + (bit >> 3)] >> (bit & 7)) & (K - 1);
    }
  };
  for (int it = 0; it < iters; ++it) {
    int seq[NSEQ];
    bool act[NSEQ];
#pragma unroll
    for (int x = 0; x < NSEQ; ++x) {
      const int s = slot + (it * NSEQ + x) * nsl;
      act[x] = s < p.N;
      seq[x] = act[x] ? s : p.N - 1;
    }
    double best[NSEQ][U][BT];
    int bj[NSEQ][U][BT];
    float wnext[NSEQ];  // each step's weight, loaded one step ahead
#pragma unroll
    for (int x = 0; x < NSEQ; ++x) wnext[x] = __ldg(p.w + static_cast<size_t>(seq[x]) * n);
    fbk::Pipe<CL, NSEQ> pipe;

    auto block = [&](auto xc, int t) {
      constexpr int X = decltype(xc)::value;
      const double wt = static_cast<double>(wnext[X]);
      if (t + 1 < n) wnext[X] = __ldg(p.w + static_cast<size_t>(seq[X]) * n + t + 1);
      if (t > 0) xwait(X, t & 1);
      const bool write = t + 1 < n;
      if (write) xarm(X, (t + 1) & 1);
      const double* vr = bufV(X, t & 1);
      double a[U][JT];
#pragma unroll
      for (int u = 0; u < U; ++u)
#pragma unroll
        for (int jj = 0; jj < JT; ++jj) a[u][jj] = (t == 0) ? 0.0 : vr[tm.a_read_off(u, jj)];
#pragma unroll
      for (int u = 0; u < U; ++u)
#pragma unroll
        for (int bb = 0; bb < BT; ++bb) {
          double bv = -DBL_MAX;
          int bjj = 0;
#pragma unroll
          for (int jj = 0; jj < JT; ++jj) {
            const double d = __dsub_rn(wt, cpd[u][jj][bb]);
            const double v = __dadd_rn(a[u][jj], -__dmul_rn(d, d));
            if (jj == 0 || v > bv) {
              bv = v;
              bjj = tm.j0 + jj;
            }
          }
          if constexpr (K >= 8) {
#pragma unroll
            for (int o = TL::NBT; o < TL::TPU; o <<= 1) {
              const double ov = __shfl_xor_sync(kFullMask, bv, o);
              const int oj = __shfl_xor_sync(kFullMask, bjj, o);
              if (ov > bv || (ov == bv && oj < bjj)) {
                bv = ov;
                bjj = oj;
              }
            }
          }
          best[X][u][bb] = bv;
          bj[X][u][bb] = bjj;
        }
      if (write && tm.a_writer) {
        double* vw = bufV(X, (t + 1) & 1);
        if (contig) {
          uint32_t r;
          int off;
          tm.a_dest(tm.a_out_index(0, 0), r, off);
          uint32_t rbar = 0, ra = 0;
          if constexpr (CL > 1) {
            rbar = mapa_u32(smem_u32(mbar(X, (t + 1) & 1)), r);
            ra = mapa_u32(smem_u32(vw + off), r);
          }
          (void)rbar;
          (void)ra;
#pragma unroll
          for (int v = 0; v < U * BT; v += 2) {
            const double o0 = best[X][v / BT][v % BT], o1 = best[X][(v + 1) / BT][(v + 1) % BT];
            if constexpr (CL == 1) {
              *reinterpret_cast<double2*>(vw + off + v) = make_double2(o0, o1);
            } else {
              st_async_v2f64(ra + 8u * v, o0, o1, rbar);
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
              if constexpr (CL == 1) {
                vw[off] = best[X][u][bb];
              } else {
                st_async_f64(mapa_u32(smem_u32(vw + off), r), best[X][u][bb],
                             mapa_u32(smem_u32(mbar(X, (t + 1) & 1)), r));
              }
            }
        }
      }
      pipe.before_stores();
      if (wk_act[X] && is_walker(X)) walk_step(X, n - 1 - t);  // previous sequence of this slot
      if (write && tm.a_writer) {
        // the thread's groups a_out_index(u, bb) are NB consecutive groups: NB * KB bits
        uint8_t* brow = bp_buf(X, it) + static_cast<size_t>(t + 1) * row_bytes + ((tm.a_out_index(0, 0) * KB) >> 3);
        uint32_t packed = 0;
#pragma unroll
        for (int v = 0; v < NB; ++v) packed |= static_cast<uint32_t>(bj[X][v / BT][v % BT]) << (KB * v);
        if constexpr (NB * KB == 8) {
          *brow = static_cast<uint8_t>(packed);
        } else {
          *reinterpret_cast<uint16_t*>(brow) = static_cast<uint16_t>(packed);
        }
      }
      pipe.after_stores();
    };
    for (int t = 0; t < n; ++t) {
      block(std::integral_constant<int, 0>{}, t);
      if constexpr (NSEQ == 2) block(std::integral_constant<int, 1>{}, t);
    }
    pipe.drain();

    // End state of each sequence: the largest final metric, lowest state on ties.
    int send[NSEQ];
    double vend[NSEQ];
#pragma unroll
    for (int x = 0; x < NSEQ; ++x) {
      double vb = -DBL_MAX;
      int sb = S;  // S marks "no candidate"; the reductions keep a valid state when one exists
      if (tm.a_writer) {
#pragma unroll
        for (int u = 0; u < U; ++u)
#pragma unroll
          for (int bb = 0; bb < BT; ++bb) {
            const int st = (bj[x][u][bb] << (L - k)) | tm.a_out_index(u, bb);
            if (sb == S || best[x][u][bb] > vb || (best[x][u][bb] == vb && st < sb)) {
              vb = best[x][u][bb];
              sb = st;
            }
          }
      }
      for (int o = tm.width >> 1; o > 0; o >>= 1) {
        const double ov = __shfl_xor_sync(kFullMask, vb, o);
        const int os = __shfl_xor_sync(kFullMask, sb, o);
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
        team_sync<CL>();  // the scratch is reused by the next sequence
      }
      // Non-finite metrics (NaN inputs) can leave no comparable candidate: keep the walk in range.
      if (sb < 0 || sb >= S) sb = 0;
      send[x] = sb;
      vend[x] = vb;
    }
    // Every thread's backpointer stores are visible to the walkers after this
    // barrier; they walk this iteration's sequences during the next one.
    team_sync<CL>();
#pragma unroll
    for (int x = 0; x < NSEQ; ++x) {
      if (tm.tt == 0 && act[x]) {
        if (!isfinite(vend[x])) atomicOr(p.status, kDevNonFinite);
        if (p.metric) p.metric[seq[x]] = vend[x];
      }
      wk_s[x] = send[x];
      wk_seq[x] = seq[x];
      wk_act[x] = act[x];
      wk_bp[x] = bp_buf(x, it);
    }
  }
  // The sequences of the last iteration are walked back here.
#pragma unroll
  for (int x = 0; x < NSEQ; ++x) {
    if (wk_act[x] && is_walker(x)) {
      for (int ti = n - 1; ti >= 0; --ti) walk_step(x, ti);
    }
  }
  if constexpr (CL > 1) cluster_sync_all();  // no CTA leaves while its shared memory may be addressed
}

}  // namespace bcjr
