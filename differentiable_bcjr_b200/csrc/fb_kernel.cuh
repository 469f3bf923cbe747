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
// Group form (an exact rewrite of the forward-backward), in base 2:
//   alpha_t(s) = phi_t(s) + A_t(s >> k),  A_{t+1}(g) = LSE_j alpha_t((j << (L-k)) | g)
//   beta_t(p)  = B_t(p & (S/K-1)),        B_{t-1}(h) = LSE_b [phi_t((h << k) | b) + B_t(((h << k) | b) & (S/K-1))]
// A sweep step is one K-term log-sum-exp per group of K states; only the S/K
// group values move between threads.
//
// Arithmetic.
//  * Every float64 value of the log2 domain carries a factor 2^128 (the
//    scaled weights and codewords 2^64, so that their squared difference
//    carries 2^128).  With that factor the low eight bits of a double's
//    exponent field are exactly a float's biased exponent, so the roundings
//    between the two formats are integer shuffles: three instructions from a
//    double exponent argument to a float, three from a float log2 back to a
//    double, none of them on the special-function pipe that runs ex2 and lg2.
//  * Emission: with c'(s) = c(s) sqrt(log2(e)/T) and w'_t likewise,
//    phi_t(s) = -(w'_t - c'(s))^2: one float64 subtract and one float64 fma
//    per state (c' stays in registers).
//  * Forward log-sum-exp of a group: its reference is the largest of its K
//    terms read from the terms' high words (a float max over the high words
//    read as floats orders them like the doubles; one three-input max per
//    three terms), plus k + 1.  Every exponent argument is then below
//    -(k + 1) + 2^-11, so the K exponentials sum to less than one and their
//    log2 is a negative normal float.
//  * Backward: the exponent is the posterior itself,
//        log2 gamma_t(s) - 1 = phi_t(s) + B_t(g_b) + A_t(h_j) - log2 Z - 1,
//    so one exponential per state yields both the marginal and the backward
//    recursion  B_{t-1}(h) = log2 sum_b 2^(log2 gamma_t - 1) - (A_t(h) - log2 Z - 1).
//  * Forward values needed by the backward sweep are kept per step (C = 1)
//    as floats relative to a per-thread reference (the high word of the
//    thread's largest value, plus one), converted with the same shuffles; the
//    backward sweep fetches them one step ahead with cp.async.  (Keeping the
//    float64 values themselves saves the conversions but moves 60 % more
//    bytes, and the backward sweep then waits on memory.)  With C > 1 only
//    every C-th step is kept (float64) and each C-segment is recomputed.
//  * The exchange buffers a sweep starts from are zero-filled (A_0 = 0,
//    B_{n-1} = 0), so every step reads them without a select.
//
// Exchange.  On a cluster, group values go straight into the shared memory of
// the CTA that reads them next step, completing on that CTA's mbarrier.  In
// the forward sweep a warp's outputs are one block of consecutive slots: they
// are staged in the sending CTA and leave as one bulk copy per warp.  In the
// backward sweep each thread's outputs go to four CTAs and leave as
// per-thread st.async stores.
//
// Schedule.  A team (thread-block cluster, one CTA, or a slice of a warp)
// keeps NSEQ sequences in flight.  With NSEQ = 2 the steps of the two
// sequences alternate and each step ends with a split cluster barrier whose
// wait is deferred past the other sequence's step, so the barrier latency
// hides behind useful work.  Global stores of a step are issued after the
// arrive, so its release never waits for them.
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
constexpr double kScale = 0x1p128;      // factor carried by every float64 log2-domain value
constexpr double kInvScale = 0x1p-128;
constexpr double kMaxScaled = 0x1p104;  // bound on |w'| and |c'| (2^40 before scaling): exponents stay < 2^91

// y = v * 2^128 with v < 0, |v| in [2^-126, 2^128): v rounded to a float (to
// nearest, ties away from zero).  Shifted left by four, the high word holds
// the exponent field's low eight bits (v's float exponent, thanks to the 2^128
// factor) followed by 24 mantissa bits; adding one and shifting back rounds
// the mantissa to 23 bits (a carry moves into the exponent, as it should), and
// the funnel shift brings in the sign bit.  (Truncating instead would bias
// every exponential upwards by half a unit in the last place, which the
// backward recursion accumulates into the unnormalised marginals.)
__device__ __forceinline__ float scaled_to_neg_float(double y) {
  const uint32_t lo = static_cast<uint32_t>(__double2loint(y));
  const uint32_t hi = static_cast<uint32_t>(__double2hiint(y));
  return __uint_as_float(__funnelshift_r(__funnelshift_l(lo, hi, 4) + 1u, 1u, 1));
}
// v a negative normal float: v * 2^128 as a double (the inverse shuffle;
// 0xB0000000 = sign + exponent re-bias 127 -> 1023 + 128 - the float sign bit
// shifted down).
__device__ __forceinline__ double neg_float_to_scaled(float v) {
  const uint32_t f = __float_as_uint(v);
  return __hiloint2double(static_cast<int>((f >> 3) + 0xB0000000u), static_cast<int>(f << 29));
}
// High word of a double read as a float.  For the values here (|x| < 2^250)
// the exponent field's top eight bits never reach 255, so these floats are
// finite and order like the doubles they come from; ties only between doubles
// that differ in the low word.
__device__ __forceinline__ float hi_key(double x) { return __int_as_float(__double2hiint(x)); }
// The double with high word `h` and a zero low word: within 2^-20 (relative)
// of every double whose key is h, towards zero.
__device__ __forceinline__ double from_key(float h) { return __hiloint2double(__float_as_int(h), 0); }
__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
// Largest key of N terms.
template <int N>
__device__ __forceinline__ float key_max(const float* h) {
  if constexpr (N == 4) {
    return fmaxf(max3(h[0], h[1], h[2]), h[3]);
  } else if constexpr (N == 2) {
    return fmaxf(h[0], h[1]);
  } else {
    float m = h[0];
#pragma unroll
    for (int i = 1; i < N; ++i) m = fmaxf(m, h[i]);
    return m;
  }
}

__device__ __forceinline__ float group_max_key(float v, int width) {
  for (int o = width >> 1; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, o));
  return v;
}
// Sum over aligned groups of `width` lanes of a pair, with packed adds.
__device__ __forceinline__ float2 group_sum2(float2 v, int width) {
  for (int o = width >> 1; o > 0; o >>= 1) {
    const float2 w = make_float2(__shfl_xor_sync(kFull, v.x, o), __shfl_xor_sync(kFull, v.y, o));
    v = __fadd2_rn(v, w);
  }
  return v;
}

// Barrier schedule of one team.  With NSEQ >= 2 on a cluster: after block b,
// wait for the phase of block b-1 (the previous sequence's block) and arrive
// for block b.  Global stores go after the arrive.
// On a cluster the exchanged data travel with st.async or bulk copies and are
// awaited on mbarriers, so this barrier orders execution only (every read of a
// buffer, and every bulk copy's read of its staging block, before the
// overwrite two steps later) and carries no memory fence.
template <int CL, int NSEQ>
struct Pipe {
  bool pending = false;
  __device__ __forceinline__ void before_stores() {
    if constexpr (CL == 1) {
      __syncthreads();
    } else if constexpr (NSEQ == 1) {
      cluster_arrive_relaxed();
    } else {
      if (pending) cluster_wait_plain();
      cluster_arrive_relaxed();
      pending = true;
    }
  }
  __device__ __forceinline__ void after_stores() {
    if constexpr (CL > 1 && NSEQ == 1) cluster_wait_plain();
  }
  __device__ __forceinline__ void drain() {
    if constexpr (CL > 1 && NSEQ >= 2) {
      if (pending) cluster_wait_plain();
      pending = false;
    }
  }
};

// f(integral_constant<int, I>) for I = 0 .. N-1, unrolled at compile time.
template <int I, int N>
struct SeqLoop {
  template <typename F>
  __device__ __forceinline__ static void run(F&& f) {
    f(std::integral_constant<int, I>{});
    SeqLoop<I + 1, N>::run(f);
  }
};
template <int N>
struct SeqLoop<N, N> {
  template <typename F>
  __device__ __forceinline__ static void run(F&&) {}
};

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
// Team-wide maximum of a key.
template <int K, int CL>
__device__ __forceinline__ float team_max_key(const Team<K, CL>& tm, float* red, float v) {
  v = group_max_key(v, tm.width);
  if (tm.TS <= 32) return v;
  if (tm.lane == 0) {
#pragma unroll
    for (int r = 0; r < CL; ++r) team_store<CL>(red, r, tm.warp_in_team, v);
  }
  team_sync<CL>();
  float m = -FLT_MAX;
  for (int i = 0; i < tm.wpt; ++i) m = fmaxf(m, red[i]);
  team_sync<CL>();
  return m;
}

}  // namespace fbk

template <int K, int CL, bool ADJ, int NSEQ, int NTB>
__global__ void __launch_bounds__(NTB, 1) fb_kernel(const FBParams p) {
  using TL = Tile<K>;
  constexpr int U = TL::U, JT = TL::JT, BT = TL::BT, NV = U * JT;
  // A cluster team fills its cluster exactly (S / 16 = CL * NTB threads), so
  // the trellis size is a compile-time constant there and every index below
  // folds to immediates; single-CTA teams take it from the parameters.
  constexpr int kLog2K = K == 2 ? 1 : K == 4 ? 2 : K == 8 ? 3 : 4;
  constexpr int kLc = CL > 1 ? ilog2_constexpr(kStatesPerThread * CL * NTB) : 0;
  const int L = kLc ? kLc : p.L;
  constexpr int k = kLog2K;
  // For K <= 4 every thread writes its forward and its backward outputs.
  constexpr bool kAllWrite = K <= 4;
  const int n = p.n, C = p.C;
  const bool alias = (C == 1);
  const int S = 1 << L;
  const int TS = S / kStatesPerThread;
  const int NT = CL > 1 ? NTB : static_cast<int>(blockDim.x);
  const int tpc = (CL == 1 && TS < NT) ? NT / TS : 1;
  const int team_in_cta = (tpc > 1) ? static_cast<int>(threadIdx.x) / TS : 0;
  Team<K, CL> tm;
  tm.init(L, k, team_in_cta * TS);
  const int slot = (CL > 1) ? static_cast<int>(blockIdx.x) / CL : static_cast<int>(blockIdx.x) * tpc + team_in_cta;
  const int GL = tm.GL;
  // The K (k <= 2: all U*K) outputs of a forward step land in consecutive slots of one CTA.
  const bool contig = (K <= 4) && (L >= 3 * k);
  // Forward reference offset: k + 1 above the largest term's key.
  constexpr double kRefOff = static_cast<double>(k + 1) * fbk::kScale;

  extern __shared__ __align__(16) unsigned char smem_raw[];
  // In the forward sweep, cluster teams with K <= 4 and up to two sequences in
  // flight stage a warp's outgoing values in their own shared memory and send
  // them as one bulk copy instead of a store per thread (the adjoint only with
  // C = 1: with C > 1 its backward buffers leave no room).  The backward
  // sweep keeps per-thread stores: a warp's outputs there form one block per
  // output row, and four staged copies per step measured slower than the
  // stores.
  constexpr bool kBulk = CL > 1 && K <= 4 && NSEQ <= 2;
  const bool xst_on = kBulk && (!ADJ || alias);
  const FBSmem lay = fb_smem_layout(GL, NT, NV, NSEQ, ADJ, alias, tpc, xst_on);
  unsigned char* team_base = smem_raw + static_cast<size_t>(team_in_cta) * lay.per_team;
  float* red = reinterpret_cast<float*>(smem_raw + lay.red);
  float* redk = reinterpret_cast<float*>(smem_raw + lay.red) + 256;

  // Codewords of the thread's 16 states: scaled float64 in registers (the
  // emission), float in shared memory (the float32 sums of the backward
  // sweep): keeping the floats out of registers leaves the forward sweep
  // more registers for independent work.
  const double sqsc = p.sqsc;  // sqrt(log2(e) / T) * 2^64
  static_assert(BT % 2 == 0, "state pairs along b");
  // (c(s_b), c(s_b+1)) float pairs in shared memory, pair e of thread i at [e][i]
  float2* cfs = reinterpret_cast<float2*>(smem_raw + lay.cf) + threadIdx.x;
  auto cf2 = [&](int u, int jj, int bp) -> float2 { return cfs[((u * JT + jj) * (BT / 2) + bp) * NT]; };
  double cp[U][JT][BT];
  bool bad_cb = false;
#pragma unroll
  for (int u = 0; u < U; ++u)
#pragma unroll
    for (int jj = 0; jj < JT; ++jj)
#pragma unroll
      for (int bb = 0; bb < BT; ++bb) {
        const float cv = __ldg(p.codebook + tm.state(u, jj, bb));
        float* slot = reinterpret_cast<float*>(cfs + ((u * JT + jj) * (BT / 2) + bb / 2) * NT);
        slot[bb & 1] = cv;
        cp[u][jj][bb] = static_cast<double>(cv) * sqsc;
        bad_cb |= !(fabs(cp[u][jj][bb]) <= fbk::kMaxScaled);
      }
  if (bad_cb) atomicOr(p.status, kDevNonFinite);
  float2 gc2[U][JT][BT / 2];  // codebook-gradient accumulators (halves), pairs along b
  if constexpr (ADJ) {
#pragma unroll
    for (int u = 0; u < U; ++u)
#pragma unroll
      for (int jj = 0; jj < JT; ++jj)
#pragma unroll
        for (int bb = 0; bb < BT / 2; ++bb) gc2[u][jj][bb] = make_float2(0.f, 0.f);
  }

  // Exchange mbarriers (cluster teams): per sequence in flight, one per
  // buffer set (forward, backward) and parity; armed each step by thread 0
  // with the bytes the CTA is about to receive.  With C == 1 the backward
  // sweep reuses the forward buffers and their mbarriers.
  const int setB = alias ? 0 : 1;
  const uint32_t xbytes = static_cast<uint32_t>(GL) * (ADJ ? 12u : 8u);
  auto mbar = [&](int X, int set, int par) {
    return reinterpret_cast<uint64_t*>(team_base + static_cast<size_t>(X) * lay.per_seq + lay.mbar) + set * 2 + par;
  };
  uint32_t ph[NSEQ];  // parity of the next phase to wait for, bit (set * 2 + par)
#pragma unroll
  for (int x = 0; x < NSEQ; ++x) ph[x] = 0;
  bool timed_out = false;  // after one wait gave up, no further waits (the call's results are void)
  if constexpr (CL > 1) {
    if (threadIdx.x == 0) {
#pragma unroll
      for (int x = 0; x < NSEQ; ++x)
        for (int i = 0; i < 4; ++i) mbar_init(mbar(x, i >> 1, i & 1), 1);
      mbar_init_fence();
    }
  }
  auto xwait = [&](int X, int set, int par) {
    if constexpr (CL > 1) {
      const int bit = set * 2 + par;
      if (!timed_out) timed_out = !mbar_wait(mbar(X, set, par), (ph[X] >> bit) & 1u, p.status, kDevTimeout);
      ph[X] ^= 1u << bit;
    }
  };
  auto xarm = [&](int X, int set, int par) {
    if constexpr (CL > 1) {
      if (threadIdx.x == 0) mbar_arm(mbar(X, set, par), xbytes);
    }
  };

  // Every CTA of the cluster must be running (and its mbarriers initialised)
  // before any of them writes into another's shared memory.
  if constexpr (CL > 1) {
    cluster_sync_all();
    if (p.probe_wait_cycles > 0) {
      // Testing aid: one bounded wait on a barrier nothing arrives at, before
      // any exchange has started; it gives up and reports the timeout.
      mbar_wait(mbar(0, 0, 0), 0u, p.status, kDevTimeout, p.probe_wait_cycles);
      cluster_sync_all();
      return;
    }
  }

  const int tvo = tm.tt * NV;  // this thread's offset in a thread-private row
  const int nsl = p.num_slots;
  const int iters = (p.N + nsl * NSEQ - 1) / (nsl * NSEQ);

  // Per-sequence state (identical in every thread of the team).
  struct Seq {
    int seq;
    bool act;
    bool bad;   // an input weight was not finite or out of range
    double K0;  // -(log2 Z + 1), scaled
    float Dc;   // backward call: E[sum_t g_t (c(s_t) - w_hat_t)]
    float wq, gq, hq;  // the next step's weight (and upstream gradient, soft codeword), loaded one step ahead
  };

  for (int it = 0; it < iters; ++it) {
    Seq sq[NSEQ];
#pragma unroll
    for (int x = 0; x < NSEQ; ++x) {
      const int s = slot + (it * NSEQ + x) * nsl;
      sq[x].act = s < p.N;
      sq[x].seq = sq[x].act ? s : p.N - 1;
      sq[x].bad = false;
      sq[x].K0 = 0.0;
      sq[x].Dc = 0.f;
    }
    // Inputs of sequence X at step t, loaded one step before they are used.
    auto load_inputs = [&](Seq& c, int t) {
      const size_t o = static_cast<size_t>(c.seq) * n + t;
      c.wq = __ldg(p.w + o);
      if constexpr (ADJ) {
        c.gq = __ldg(p.g + o);
        c.hq = __ldg(p.what_in + o);
      }
    };
#pragma unroll
    for (int x = 0; x < NSEQ; ++x) load_inputs(sq[x], 0);
    fbk::Pipe<CL, NSEQ> pipe;

    // Zero buffer `par` of the group-value exchange area at byte offset `offA`
    // (and of the adjoint accumulators at `offF`) for every sequence in flight:
    // the part this CTA holds.
    auto zero_exchange = [&](uint32_t offA, uint32_t offF, int par) {
      const int nt_team = CL > 1 ? NT : TS;
      const int tid = CL > 1 ? static_cast<int>(threadIdx.x) : tm.tt;
#pragma unroll
      for (int x = 0; x < NSEQ; ++x) {
        unsigned char* sb = team_base + static_cast<size_t>(x) * lay.per_seq;
        double* zA = reinterpret_cast<double*>(sb + offA) + par * GL;
        float* zF = reinterpret_cast<float*>(sb + offF) + par * GL;
        for (int i = tid; i < GL; i += nt_team) {
          zA[i] = 0.0;
          if constexpr (ADJ) zF[i] = 0.f;
        }
      }
    };

    // Forward step of sequence X at step t: reads A_t (and F~_t) from the
    // exchange buffers, or from a0/f0 when given; when `write` is set, writes
    // A_{t+1} (and F~_{t+1}) to the readers' exchange buffers.  Leaves the
    // inputs in a / f.
    auto forward_step = [&](auto xc, int t, const double* a0, const float* f0, bool write, double* a, float* f,
                            float wt, float gt, float gw) {
      constexpr int X = decltype(xc)::value;
      Seq& c = sq[X];
      unsigned char* sb = team_base + static_cast<size_t>(X) * lay.per_seq;
      const double* exA_r = reinterpret_cast<const double*>(sb + lay.exA) + (t & 1) * GL;
      double* exA_w = reinterpret_cast<double*>(sb + lay.exA) + ((t + 1) & 1) * GL;
      const float* exF_r = reinterpret_cast<const float*>(sb + lay.exF) + (t & 1) * GL;
      float* exF_w = reinterpret_cast<float*>(sb + lay.exF) + ((t + 1) & 1) * GL;
      if (!a0 && t > 0) xwait(X, 0, t & 1);
      if (write) xarm(X, 0, (t + 1) & 1);
#pragma unroll
      for (int u = 0; u < U; ++u)
#pragma unroll
        for (int jj = 0; jj < JT; ++jj) {
          if (a0) {
            a[u * JT + jj] = a0[u * JT + jj];
            if constexpr (ADJ) f[u * JT + jj] = f0[u * JT + jj];
          } else {
            a[u * JT + jj] = exA_r[tm.a_read_off(u, jj)];
            if constexpr (ADJ) f[u * JT + jj] = exF_r[tm.a_read_off(u, jj)];
          }
        }
      if (!write) return;
      const double wp = static_cast<double>(wt) * sqsc;
      c.bad |= !(fabs(wp) <= fbk::kMaxScaled);
      double outs[U][BT];
      float fos[U][BT];
      // Two groups (b, b+1) at a time, so that the float32 sums run on packed
      // f32x2 instructions.  Adjoint: num_b = sum_j e_jb (F~_j + g c_jb - g w_hat)
      // = sum_j e_jb F~_j + g sum_j e_jb c_jb - g w_hat s_b.
      const float2 gt2 = make_float2(gt, gt), ngw2 = make_float2(-gw, -gw);
#pragma unroll
      for (int u = 0; u < U; ++u) {
#pragma unroll
        for (int bp = 0; bp < BT / 2; ++bp) {
          const int b0 = 2 * bp, b1 = b0 + 1;
          double x0[JT], x1[JT];
          float h0[JT], h1[JT];
#pragma unroll
          for (int jj = 0; jj < JT; ++jj) {
            const double d0 = wp - cp[u][jj][b0], d1 = wp - cp[u][jj][b1];
            x0[jj] = fma(-d0, d0, a[u * JT + jj]);
            x1[jj] = fma(-d1, d1, a[u * JT + jj]);
            h0[jj] = fbk::hi_key(x0[jj]);
            h1[jj] = fbk::hi_key(x1[jj]);
          }
          float k0 = fbk::key_max<JT>(h0), k1 = fbk::key_max<JT>(h1);
          if constexpr (K >= 8) {
#pragma unroll
            for (int o = TL::NBT; o < TL::TPU; o <<= 1) {
              k0 = fmaxf(k0, __shfl_xor_sync(fbk::kFull, k0, o));
              k1 = fmaxf(k1, __shfl_xor_sync(fbk::kFull, k1, o));
            }
          }
          const double ref0 = fbk::from_key(k0) + kRefOff, ref1 = fbk::from_key(k1) + kRefOff;
          float2 s2 = make_float2(0.f, 0.f), na2 = make_float2(0.f, 0.f), nc2 = make_float2(0.f, 0.f);
#pragma unroll
          for (int jj = 0; jj < JT; ++jj) {
            const float2 e = make_float2(ex2f(fbk::scaled_to_neg_float(x0[jj] - ref0)),
                                         ex2f(fbk::scaled_to_neg_float(x1[jj] - ref1)));
            s2 = __fadd2_rn(s2, e);
            if constexpr (ADJ) {
              const float fj = f[u * JT + jj];
              na2 = __ffma2_rn(e, make_float2(fj, fj), na2);
              nc2 = __ffma2_rn(e, cf2(u, jj, bp), nc2);
            }
          }
          if constexpr (K >= 8) {
#pragma unroll
            for (int o = TL::NBT; o < TL::TPU; o <<= 1) {
              s2.x += __shfl_xor_sync(fbk::kFull, s2.x, o);
              s2.y += __shfl_xor_sync(fbk::kFull, s2.y, o);
              if constexpr (ADJ) {
                na2.x += __shfl_xor_sync(fbk::kFull, na2.x, o);
                na2.y += __shfl_xor_sync(fbk::kFull, na2.y, o);
                nc2.x += __shfl_xor_sync(fbk::kFull, nc2.x, o);
                nc2.y += __shfl_xor_sync(fbk::kFull, nc2.y, o);
              }
            }
          }
          // s < 1: its log2 is a negative normal float
          outs[u][b0] = fbk::neg_float_to_scaled(lg2f(s2.x)) + ref0;
          outs[u][b1] = fbk::neg_float_to_scaled(lg2f(s2.y)) + ref1;
          if constexpr (ADJ) {
            const float2 num2 = __ffma2_rn(ngw2, s2, __ffma2_rn(gt2, nc2, na2));
            fos[u][b0] = num2.x * rcpf(s2.x);
            fos[u][b1] = num2.y * rcpf(s2.y);
          }
        }
      }
      if (!kAllWrite && !tm.a_writer) return;
      const uint32_t bar_l = smem_u32(mbar(X, 0, (t + 1) & 1));
      if (contig) {
        uint32_t r;
        int off;
        tm.a_dest(tm.a_out_index(0, 0), r, off);
        uint32_t rbar = 0, ra_ = 0, rf_ = 0;
        if constexpr (CL > 1) {
          rbar = mapa_u32(bar_l, r);
          ra_ = mapa_u32(smem_u32(exA_w + off), r);
          if constexpr (ADJ) rf_ = mapa_u32(smem_u32(exF_w + off), r);
        }
        if (xst_on) {
          // The warp's 32 x U*BT values are consecutive slots of one CTA: stage
          // them in the same order (slot parity and sequence of their own) and
          // let lane 0 copy the block.  The staging slot is rewritten two steps
          // later, after the barrier that follows every reader's wait for it.
          const int sidx = (X * 2 + ((t + 1) & 1)) * GL + threadIdx.x * (U * BT);
          double* stg = reinterpret_cast<double*>(smem_raw + lay.xst) + sidx;
          float* stgF = reinterpret_cast<float*>(smem_raw + lay.xstF) + sidx;
#pragma unroll
          for (int v = 0; v < U * BT; v += 2)
            *reinterpret_cast<double2*>(stg + v) = make_double2(outs[v / BT][v % BT], outs[(v + 1) / BT][(v + 1) % BT]);
          if constexpr (ADJ) {
#pragma unroll
            for (int v = 0; v < U * BT; v += 4)
              *reinterpret_cast<float4*>(stgF + v) =
                  make_float4(fos[v / BT][v % BT], fos[(v + 1) / BT][(v + 1) % BT], fos[(v + 2) / BT][(v + 2) % BT],
                              fos[(v + 3) / BT][(v + 3) % BT]);
          }
          async_proxy_fence();
          __syncwarp();
          if (tm.lane == 0) {
            bulk_copy_s2c(ra_, smem_u32(stg), 32u * U * BT * 8u, rbar);
            if constexpr (ADJ) bulk_copy_s2c(rf_, smem_u32(stgF), 32u * U * BT * 4u, rbar);
          }
          return;
        }
#pragma unroll
        for (int v = 0; v < U * BT; v += 2) {
          const double o0 = outs[v / BT][v % BT], o1 = outs[(v + 1) / BT][(v + 1) % BT];
          if constexpr (CL == 1) {
            *reinterpret_cast<double2*>(exA_w + off + v) = make_double2(o0, o1);
            if constexpr (ADJ)
              *reinterpret_cast<float2*>(exF_w + off + v) =
                  make_float2(fos[v / BT][v % BT], fos[(v + 1) / BT][(v + 1) % BT]);
          } else {
            st_async_v2f64(ra_ + 8u * v, o0, o1, rbar);
            if constexpr (ADJ) {  // four accumulators per store (U * BT is 4 or 8)
              if (v % 4 == 0)
                st_async_v4f32(rf_ + 4u * v, fos[v / BT][v % BT], fos[(v + 1) / BT][(v + 1) % BT],
                               fos[(v + 2) / BT][(v + 2) % BT], fos[(v + 3) / BT][(v + 3) % BT], rbar);
            }
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
              exA_w[off] = outs[u][bb];
              if constexpr (ADJ) exF_w[off] = fos[u][bb];
            } else {
              const uint32_t rbar = mapa_u32(bar_l, r);
              st_async_f64(mapa_u32(smem_u32(exA_w + off), r), outs[u][bb], rbar);
              if constexpr (ADJ) st_async_f32(mapa_u32(smem_u32(exF_w + off), r), fos[u][bb], rbar);
            }
          }
      }
    };

    // Checkpoint row of the forward values A_t (and F~_t): floats relative to
    // the thread's reference R = (largest value's high word) + 1, and that high word.
    auto store_checkpoint = [&](const double* a, const float* f, size_t row_index, size_t lane_id) {
      float* ckrow = p.ck + lane_id * p.ck_stride + row_index * p.row + tvo;
      uint32_t* ckkey = p.ckR + lane_id * p.ckR_stride + row_index * TS + tm.tt;
      float hk[NV];
#pragma unroll
      for (int v = 0; v < NV; ++v) hk[v] = fbk::hi_key(a[v]);
      const float key = fbk::key_max<NV>(hk);
      const double R1 = fbk::from_key(key) + fbk::kScale;
#pragma unroll
      for (int v = 0; v < NV; v += 4) {
        *reinterpret_cast<float4*>(ckrow + v) = make_float4(
            fbk::scaled_to_neg_float(a[v] - R1), fbk::scaled_to_neg_float(a[v + 1] - R1),
            fbk::scaled_to_neg_float(a[v + 2] - R1), fbk::scaled_to_neg_float(a[v + 3] - R1));
        if constexpr (ADJ) {
          float* ckrowF = p.ckF + lane_id * p.ck_stride + row_index * p.row + tvo;
          *reinterpret_cast<float4*>(ckrowF + v) = make_float4(f[v], f[v + 1], f[v + 2], f[v + 3]);
        }
      }
      *ckkey = __float_as_uint(key);
    };

    // ---------------- forward sweep ----------------
    auto alpha_block = [&](auto xc, int t) {
      constexpr int X = decltype(xc)::value;
      const size_t lane_id = static_cast<size_t>(slot) * NSEQ + X;
      Seq& c = sq[X];
      const float wt = c.wq, gt = ADJ ? c.gq : 0.f, gw = ADJ ? c.gq * c.hq : 0.f;
      if (t + 1 < n) load_inputs(c, t + 1);
      double a[NV];
      float f[NV];
      forward_step(xc, t, nullptr, nullptr, true, a, f, wt, gt, gw);
      pipe.before_stores();
      // ---- this step's global stores (outside the barrier's release) ----
      if (C == 1) {
        store_checkpoint(a, f, static_cast<size_t>(t), lane_id);
      } else if (t % C == 0) {  // exact float64 forward values at the segment starts
        double* row = p.ck64 + lane_id * p.ck64_stride + static_cast<size_t>(t / C) * p.row + tvo;
        float* rowF = ADJ ? p.ckF64 + lane_id * p.ck64_stride + static_cast<size_t>(t / C) * p.row + tvo : nullptr;
#pragma unroll
        for (int u = 0; u < U; ++u)
#pragma unroll
          for (int jj = 0; jj < JT; ++jj) {
            row[u * JT + jj] = a[u * JT + jj];
            if constexpr (ADJ) rowF[u * JT + jj] = f[u * JT + jj];
          }
      }
      pipe.after_stores();
    };

    // A_0 = 0 (and F~_0 = 0): zero-fill the buffers step 0 reads.  Every read
    // of them in the previous sequence ended before the team barrier that
    // closed it, and no CTA writes them again before this CTA has passed the
    // barrier of its own step 0.
    zero_exchange(lay.exA, lay.exF, 0);
    if constexpr (CL > 1) {
      __syncthreads();
    } else {
      team_sync<CL>();
    }
    for (int t = 0; t < n; ++t) {
      fbk::SeqLoop<0, NSEQ>::run([&](auto xc) { alpha_block(xc, t); });
    }
    pipe.drain();

    // log2 Z = log2 sum_g 2^{A_n(g)};  D = E[sum_t g_t (c(s_t) - w_hat_t)] (backward call).
    auto finish_forward = [&](auto xc) {
      constexpr int X = decltype(xc)::value;
      Seq& c = sq[X];
      unsigned char* sb = team_base + static_cast<size_t>(X) * lay.per_seq;
      const double* exA_r = reinterpret_cast<const double*>(sb + lay.exA) + (n & 1) * GL;
      const float* exF_r = reinterpret_cast<const float*>(sb + lay.exF) + (n & 1) * GL;
      xwait(X, 0, n & 1);
      double av[U][JT];
      float key = -FLT_MAX;
#pragma unroll
      for (int u = 0; u < U; ++u)
#pragma unroll
        for (int jj = 0; jj < JT; ++jj) {
          av[u][jj] = exA_r[tm.a_read_off(u, jj)];
          if (kAllWrite || tm.b_writer) key = fmaxf(key, fbk::hi_key(av[u][jj]));  // one reader per group value
        }
      const double Rt = fbk::from_key(fbk::team_max_key(tm, redk, key));
      float s1 = 0.f, s2 = 0.f;
      if (kAllWrite || tm.b_writer) {
#pragma unroll
        for (int u = 0; u < U; ++u)
#pragma unroll
          for (int jj = 0; jj < JT; ++jj) {
            const float e = ex2f(static_cast<float>((av[u][jj] - Rt) * fbk::kInvScale));
            s1 += e;
            if constexpr (ADJ) s2 = fmaf(e, exF_r[tm.a_read_off(u, jj)], s2);
          }
      }
      const double S1 = fbk::team_sum(tm, red, s1);
      const double S2 = ADJ ? fbk::team_sum(tm, red + 128, s2) : 0.0;
      const double log2Z = Rt * fbk::kInvScale + log2(S1);  // unscaled
      c.K0 = -(log2Z + 1.0) * fbk::kScale;
      c.Dc = ADJ ? static_cast<float>(S2 / S1) : 0.f;
      if (tm.tt == 0 && c.act) {
        const bool ok = isfinite(log2Z) && !c.bad;
        if (!ok) atomicOr(p.status, kDevNonFinite);
        if constexpr (!ADJ) {
          if (p.log_z) p.log_z[c.seq] = ok ? static_cast<float>(log2Z * 0.69314718055994530942) : NAN;
        }
      }
    };
    fbk::SeqLoop<0, NSEQ>::run([&](auto xc) { finish_forward(xc); });
    team_sync<CL>();
    // B_{n-1} = 0 (and B~_{n-1} = 0): zero-fill the buffers step n-1 reads; the
    // forward sweep's last use of them ended before the barrier above.
    zero_exchange(lay.exB, lay.exBt, (n - 1) & 1);
    if constexpr (CL > 1) {
      __syncthreads();
    } else {
      team_sync<CL>();
    }

    // ---------------- backward sweep ----------------
    // C > 1: recompute the forward values of the segment [t0, t1] into the ring
    // (rows 0 .. t1-t0, same format as the C = 1 rows).
    auto recompute_segment = [&](int t0, int t1) {
      for (int tp = t0; tp <= t1; ++tp) {
        auto one = [&](auto xc) {
          constexpr int X = decltype(xc)::value;
          const size_t lane_id = static_cast<size_t>(slot) * NSEQ + X;
          const double* c64 = p.ck64 + lane_id * p.ck64_stride + static_cast<size_t>(t0 / C) * p.row + tvo;
          const float* cF64 =
              ADJ ? p.ckF64 + lane_id * p.ck64_stride + static_cast<size_t>(t0 / C) * p.row + tvo : nullptr;
          const size_t o = static_cast<size_t>(sq[X].seq) * n + tp;
          const float wt = __ldg(p.w + o);
          const float gt = ADJ ? __ldg(p.g + o) : 0.f, gw = ADJ ? gt * __ldg(p.what_in + o) : 0.f;
          double a[NV];
          float f[NV];
          forward_step(xc, tp, tp == t0 ? c64 : nullptr, tp == t0 ? cF64 : nullptr, tp < t1, a, f, wt, gt, gw);
          store_checkpoint(a, f, static_cast<size_t>(tp - t0), lane_id);
        };
        fbk::SeqLoop<0, NSEQ>::run(one);
        team_sync<CL>();
      }
    };

    // Staging of the stored forward values of one step (C == 1), one slot per
    // sequence in flight: NV floats, the reference word and (adjoint) NV
    // forward adjoint accumulators.  A block consumes its slot into registers
    // before it refills it for the step below, so one slot suffices; the
    // refill has NSEQ blocks to land.
    auto stage_index = [&](int X) { return static_cast<size_t>(X) * NT + threadIdx.x; };
    auto prefetch_row = [&](int X, int t_row) {
      const size_t lane_id = static_cast<size_t>(slot) * NSEQ + X;
      const size_t idx = stage_index(X);
      float* sf = reinterpret_cast<float*>(smem_raw + lay.stage) + idx * NV;
      uint32_t* sK = reinterpret_cast<uint32_t*>(smem_raw + lay.stageK) + idx;
      const float* src = p.ck + lane_id * p.ck_stride + static_cast<size_t>(t_row) * p.row + tvo;
#pragma unroll
      for (int v = 0; v < NV; v += 4) {
        cp_async16(sf + v, src + v);
        if constexpr (ADJ) {
          float* sF = reinterpret_cast<float*>(smem_raw + lay.stageF) + idx * NV;
          const float* srcF = p.ckF + lane_id * p.ck_stride + static_cast<size_t>(t_row) * p.row + tvo;
          cp_async16(sF + v, srcF + v);
        }
      }
      cp_async4(sK, p.ckR + lane_id * p.ckR_stride + static_cast<size_t>(t_row) * TS + tm.tt);
    };

    auto beta_block = [&](auto xc, int t) {
      constexpr int X = decltype(xc)::value;
      Seq& c = sq[X];
      unsigned char* sb = team_base + static_cast<size_t>(X) * lay.per_seq;
      const size_t lane_id = static_cast<size_t>(slot) * NSEQ + X;
      const double* exB_r = reinterpret_cast<const double*>(sb + lay.exB) + (t & 1) * GL;
      double* exB_w = reinterpret_cast<double*>(sb + lay.exB) + ((t + 1) & 1) * GL;  // (t-1) & 1
      const float* exBt_r = reinterpret_cast<const float*>(sb + lay.exBt) + (t & 1) * GL;
      float* exBt_w = reinterpret_cast<float*>(sb + lay.exBt) + ((t + 1) & 1) * GL;
      // r_j = A_t(h_j) - log2 Z - 1 (scaled), so that log2 gamma_t(s) - 1 = phi_t(s) + B_t(g_b) + r_j
      double rp[NV];
      float fa[NV];
      if (C == 1) {
        const size_t idx = stage_index(X);
        cp_async_wait<NSEQ - 1>();  // this sequence's row, committed NSEQ groups ago
        const float* sf = reinterpret_cast<const float*>(smem_raw + lay.stage) + idx * NV;
        const uint32_t* sK = reinterpret_cast<const uint32_t*>(smem_raw + lay.stageK) + idx;
        const double RK = fbk::from_key(__uint_as_float(*sK)) + (fbk::kScale + c.K0);
#pragma unroll
        for (int v = 0; v < NV; v += 4) {
          const float4 q4 = *reinterpret_cast<const float4*>(sf + v);
          rp[v] = fbk::neg_float_to_scaled(q4.x) + RK;
          rp[v + 1] = fbk::neg_float_to_scaled(q4.y) + RK;
          rp[v + 2] = fbk::neg_float_to_scaled(q4.z) + RK;
          rp[v + 3] = fbk::neg_float_to_scaled(q4.w) + RK;
          if constexpr (ADJ) {
            const float* sF = reinterpret_cast<const float*>(smem_raw + lay.stageF) + idx * NV;
            const float4 f4 = *reinterpret_cast<const float4*>(sF + v);
            fa[v] = f4.x;
            fa[v + 1] = f4.y;
            fa[v + 2] = f4.z;
            fa[v + 3] = f4.w;
          }
        }
        if (t >= 1) prefetch_row(X, t - 1);  // the slot's values are in registers now
        cp_async_commit();
      } else {
        const int t0 = t - (t % C);
        const size_t ri = static_cast<size_t>(t - t0);
        const float* ring = p.ck + lane_id * p.ck_stride + ri * p.row + tvo;
        const double RK =
            fbk::from_key(__uint_as_float(p.ckR[lane_id * p.ckR_stride + ri * TS + tm.tt])) + (fbk::kScale + c.K0);
#pragma unroll
        for (int v = 0; v < NV; ++v) {
          rp[v] = fbk::neg_float_to_scaled(ring[v]) + RK;
          if constexpr (ADJ) fa[v] = p.ckF[lane_id * p.ck_stride + ri * p.row + tvo + v];
        }
      }
      const float wt = c.wq;
      const double wp = static_cast<double>(wt) * sqsc;
      const float gt = ADJ ? c.gq : 0.f, gw = ADJ ? c.gq * c.hq : 0.f;
      if (t >= 1) load_inputs(c, t - 1);
      // incoming B_t at the thread's successor groups (q << k) | b
      if (t < n - 1) xwait(X, setB, t & 1);
      if (t >= 1) xarm(X, setB, (t + 1) & 1);
      const uint32_t bar_l = smem_u32(mbar(X, setB, (t + 1) & 1));
      double bv[U][BT];
      float2 ub2[U][BT / 2];  // adjoint: B~_t(g_b) - g w_hat, pairs along b
#pragma unroll
      for (int u = 0; u < U; ++u)
#pragma unroll
        for (int bb = 0; bb < BT; ++bb) bv[u][bb] = exB_r[tm.b_read_off(u, bb)];
      if constexpr (ADJ) {
#pragma unroll
        for (int u = 0; u < U; ++u)
#pragma unroll
          for (int bp = 0; bp < BT / 2; ++bp)
            ub2[u][bp] = make_float2(exBt_r[tm.b_read_off(u, 2 * bp)] - gw, exBt_r[tm.b_read_off(u, 2 * bp + 1)] - gw);
      }
      // Inactive (padding) sequences contribute nothing to the codebook gradient.
      const float actf = c.act ? 1.f : 0.f;
      const float gta = gt * actf;
      const float m2T = -p.two_over_T * actf;
      const float twa = p.two_over_T * wt * actf;
      const float2 gt2 = make_float2(gt, gt), gta2 = make_float2(gta, gta);
      const float2 m2T2 = make_float2(m2T, m2T), twa2 = make_float2(twa, twa);
      float2 acc02 = make_float2(0.f, 0.f), acc12 = make_float2(0.f, 0.f);
      float* mrow = (!ADJ && p.marginals && c.act)
                        ? p.marginals + (static_cast<size_t>(c.seq) * n + t) * static_cast<size_t>(S)
                        : nullptr;
      const bool send = t >= 1;
      // K = 4 cluster teams of the adjoint send the float32 accumulators of two
      // neighbouring groups (adjacent slots of one CTA) per store: the two
      // lanes of a pair swap their values of row jj and one of them stores
      // both.  (Measured: this halves the cost of the accumulators' exchange;
      // pairing the float64 outputs the same way costs more than it saves.)
      constexpr bool kPairBt = CL > 1 && K == 4 && ADJ;
      // The state loop, instantiated with and without the marginal stores so
      // that a call without marginals carries none of their addressing.
      auto states = [&](auto with_marginals) {
      constexpr bool MARG = decltype(with_marginals)::value;
#pragma unroll
      for (int u = 0; u < U; ++u) {
#pragma unroll
        for (int jj = 0; jj < JT; ++jj) {
          const double r = rp[u * JT + jj];
          const float fbase = ADJ ? fa[u * JT + jj] - c.Dc : 0.f;
          // two states per iteration: the float32 arithmetic runs on packed f32x2 instructions
          float2 s2 = make_float2(0.f, 0.f), bnum2 = make_float2(0.f, 0.f);
#pragma unroll
          for (int bp = 0; bp < BT / 2; ++bp) {
            const int b0 = 2 * bp, b1 = 2 * bp + 1;
            const float2 cv = cf2(u, jj, bp);
            const double d0 = wp - cp[u][jj][b0], d1 = wp - cp[u][jj][b1];
            const float2 e = make_float2(ex2f(fbk::scaled_to_neg_float(fma(-d0, d0, bv[u][b0] + r))),
                                         ex2f(fbk::scaled_to_neg_float(fma(-d1, d1, bv[u][b1] + r))));  // gamma_t / 2
            s2 = __fadd2_rn(s2, e);
            if constexpr (!ADJ) {
              acc02 = __ffma2_rn(e, cv, acc02);
              if constexpr (MARG) {  // gamma / 2, scaled by the step's sum after the sweep
                mrow[tm.state(u, jj, b0)] = e.x;
                mrow[tm.state(u, jj, b1)] = e.y;
              }
            } else {
              const float2 eps = __ffma2_rn(gt2, cv, ub2[u][bp]);  // g (c - w_hat) + B~_t
              const float2 ge = __fmul2_rn(e, eps);
              bnum2 = __fadd2_rn(bnum2, ge);
              const float2 psi = __ffma2_rn(e, make_float2(fbase, fbase), ge);  // psi_t / 2
              acc02 = __ffma2_rn(psi, cv, acc02);
              gc2[u][jj][bp] = __ffma2_rn(psi, __ffma2_rn(m2T2, cv, twa2), __ffma2_rn(gta2, e, gc2[u][jj][bp]));
            }
          }
          if constexpr (!ADJ) acc12 = __fadd2_rn(acc12, s2);  // this thread's states only
          float s = s2.x + s2.y, bnum = bnum2.x + bnum2.y;
          if constexpr (K >= 8) {
#pragma unroll
            for (int o = 1; o < TL::NBT; o <<= 1) {
              s += __shfl_xor_sync(fbk::kFull, s, o);
              if constexpr (ADJ) bnum += __shfl_xor_sync(fbk::kFull, bnum, o);
            }
          }
          if (send && (kAllWrite || tm.b_writer)) {
            // s = sum_b gamma / 2 <= 1/2, so its log2 is a negative normal float.  A
            // group whose posterior underflowed is raised to 2^-126: its
            // predecessors then carry at most 2^-125 in total, as negligible as 0.
            const float sc = fmaxf(s, 0x1p-126f);
            const double out = fbk::neg_float_to_scaled(lg2f(sc)) - r;
            const float bt_out = bnum * rcpf(sc);
            uint32_t rk;
            int off;
            tm.b_dest(tm.b_out_index(u, jj), rk, off);
            if constexpr (CL == 1) {
              exB_w[off] = out;
              if constexpr (ADJ) exBt_w[off] = bt_out;
            } else {
              const uint32_t rbar = mapa_u32(bar_l, rk);
              st_async_f64(mapa_u32(smem_u32(exB_w + off), rk), out, rbar);
              if constexpr (kPairBt) {
                // lanes 2i and 2i + 1 hold groups q0 - odd and q0 - odd + 1
                const int odd = tm.lane & 1;
                const float f_pair = __shfl_xor_sync(fbk::kFull, bt_out, 1);
                if (odd == (jj & 1))
                  st_async_v2f32(mapa_u32(smem_u32(exBt_w + off - odd), rk), odd ? f_pair : bt_out,
                                 odd ? bt_out : f_pair, rbar);
              } else if constexpr (ADJ) {
                st_async_f32(mapa_u32(smem_u32(exBt_w + off), rk), bt_out, rbar);
              }
            }
          }
        }
      }
      };
      if (mrow) {
        states(std::true_type{});
      } else {
        states(std::false_type{});
      }
      float2 v01;
      if constexpr (ADJ) {
        v01 = make_float2(group_sum(acc02.x + acc02.y, tm.width), 0.f);
      } else {
        v01 = fbk::group_sum2(make_float2(acc02.x + acc02.y, acc12.x + acc12.y), tm.width);
      }
      pipe.before_stores();
      if ((tm.lane & (tm.width - 1)) == 0) {
        float* pr = p.part + lane_id * p.part_stride + static_cast<size_t>(t) * 2 * tm.wpt;
        pr[tm.warp_in_team] = v01.x;
        if constexpr (!ADJ) pr[tm.wpt + tm.warp_in_team] = v01.y;
      }
      pipe.after_stores();
    };

    // stage the forward values of step n-1 before the backward pipeline starts
    if (C == 1) {
#pragma unroll
      for (int x = 0; x < NSEQ; ++x) {
        prefetch_row(x, n - 1);
        cp_async_commit();
      }
    }
#pragma unroll
    for (int x = 0; x < NSEQ; ++x) load_inputs(sq[x], n - 1);
    for (int t = n - 1; t >= 0; --t) {
      if (C > 1 && (t == n - 1 || (t + 1) % C == 0)) {
        pipe.drain();
        recompute_segment(t - (t % C), t);
      }
      fbk::SeqLoop<0, NSEQ>::run([&](auto xc) { beta_block(xc, t); });
    }
    pipe.drain();
    team_sync<CL>();
    // Per-step outputs from the per-warp partial sums (fixed order: deterministic).
#pragma unroll
    for (int x = 0; x < NSEQ; ++x) {
      if (!sq[x].act) continue;
      const size_t lane_id = static_cast<size_t>(slot) * NSEQ + x;
      for (int t = tm.tt; t < n; t += tm.TS) {
        float* pr = p.part + lane_id * p.part_stride + static_cast<size_t>(t) * 2 * tm.wpt;
        float v0 = 0.f, v1 = 0.f;
        for (int i = 0; i < tm.wpt; ++i) {
          v0 += pr[i];
          if constexpr (!ADJ) v1 += pr[tm.wpt + i];
        }
        if constexpr (!ADJ) {
          p.w_hat[static_cast<size_t>(sq[x].seq) * n + t] = v0 / v1;
          if (p.marginals) pr[0] = 1.f / v1;  // the step's normaliser, read back below
        } else {
          p.grad_w[static_cast<size_t>(sq[x].seq) * n + t] = 2.f * p.two_over_T * v0;  // v0 sums psi/2 * c
        }
      }
    }
    team_sync<CL>();
    if constexpr (!ADJ) {
      // Marginals: every state's gamma_t / 2 was stored relative to the forward
      // call's log Z, so the rounding of the fast 2^x and log2 accumulated over
      // the sweeps scales a whole step; dividing by the step's own sum (as w_hat
      // does) makes every step sum to one.
      if (p.marginals) {
#pragma unroll
        for (int x = 0; x < NSEQ; ++x) {
          if (!sq[x].act) continue;
          const size_t lane_id = static_cast<size_t>(slot) * NSEQ + x;
          for (int t = 0; t < n; ++t) {
            const float inv = p.part[lane_id * p.part_stride + static_cast<size_t>(t) * 2 * tm.wpt];
            float* mrow = p.marginals + (static_cast<size_t>(sq[x].seq) * n + t) * static_cast<size_t>(S);
#pragma unroll
            for (int u = 0; u < U; ++u)
#pragma unroll
              for (int jj = 0; jj < JT; ++jj)
#pragma unroll
                for (int bb = 0; bb < BT; ++bb) mrow[tm.state(u, jj, bb)] *= inv;
          }
        }
      }
    }
  }

  if constexpr (ADJ) {
    float* gp = p.gc_part + static_cast<size_t>(slot) * S;
#pragma unroll
    for (int u = 0; u < U; ++u)
#pragma unroll
      for (int jj = 0; jj < JT; ++jj)
#pragma unroll
        for (int bb = 0; bb < BT; ++bb)  // gc holds halves
          gp[tm.state(u, jj, bb)] = 2.f * ((bb & 1) ? gc2[u][jj][bb / 2].y : gc2[u][jj][bb / 2].x);
  }
  if constexpr (CL > 1) cluster_sync_all();  // no CTA leaves while its shared memory may be addressed
}

}  // namespace bcjr
