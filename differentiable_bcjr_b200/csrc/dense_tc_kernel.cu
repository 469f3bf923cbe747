// dense_tc_kernel.cu -- the dense (fully connected) trellis on the
// fifth-generation tensor cores (tcgen05, sm_100a): the soft codeword with its
// marginals and log Z, the vector-Jacobian product, and the rows of the
// log-transition gradient.
//
// "BCJR-QAT: A Differentiable Relaxation of Trellis-Coded Weight Quantization",
// abstract: the relaxation is a 1D Ising-like chain solved by a transfer
// matrix.  With P = exp(Lambda) (row = source state) and emission factors
// E_t(s) = 2^(phi_t(s) - m_t), phi_t(s) = -(w_t - c(s))^2 log2(e) / T and m_t the
// largest phi_t of the step, the probability-domain recursions are
//   forward   u_0 = E_0,            u_t = ((u_{t-1} P) (.) E_t) / s_{t-1},
//   backward  z_{n-1} = 1,          z_{t-1} = ((E_t (.) z_t) P^T) / sigma_t,
//   gamma_t = u_t (.) z_t / sum_s u_t(s) z_t(s),   w_hat_t = sum_s c(s) gamma_t(s),
// with s_t = sum_s u_t(s) and sigma_t = sum_s E_t(s) z_t(s): any per-row scale
// cancels in gamma, and dividing by the previous step's sum keeps every row's
// sum in (0, 1] (P is row-stochastic for the normalised Lambda, and within a
// step's column-sum spread in general).  log2 Z = sum_t m_t + sum_t log2 s_t.
// The vector-Jacobian product ("key technical innovations": exact gradients)
// runs the same recursions on a second operand per sequence, u (.) (F~ + eps)
// and v (.) (eps + B~), whose ratios to the first give the centred
// accumulators F~ and B~.
//
// Each step is one [128 x 256] x [256 x 256] contraction: a real batched
// matrix product, run here as three tf32 products (x = hi + lo, hi*hi + hi*lo +
// lo*hi: float32-level accuracy; one tf32 product would leave ~5e-4 relative
// error in a step's dominant terms).
//
// Work split.  A thread-block cluster of 4 CTAs owns a tile of 128 MMA rows:
// 128 sequences (soft codeword) or 64 sequences with their two operands on
// adjacent rows (vector-Jacobian product).  CTA r keeps K-slice r of the
// transfer matrix (input states 64r .. 64r+63, as tf32 head and tail in
// K-major core-matrix tiles, 128 KiB) resident in shared memory; its operand
// A, the same 64 states of the current vectors as head and tail, lives in
// tensor memory next to the accumulator.  The 96 MMAs of a step (4 output
// blocks of 64 states x 8 K-chunks x 3 products) give partial sums for all 256
// output states; CTA r's output states 64r .. 64r+63 are exactly its next
// K-slice, so only the partial sums cross CTAs (a reduce-scatter over
// distributed shared memory) and the operand never does.  A ninth warp issues
// the MMAs and commits the output blocks one at a time, the other CTAs'
// blocks first; each of the eight worker warps (two per tensor-memory lane
// quadrant, 32 states of a row each) sends its half of a finished block with
// st.async from registers, completing on the receiver's mbarrier, while the
// MMAs of the next block run.  The workers then add the three received halves
// to their own, scale, store and write the new operand back to tensor memory.
// The row sums for the next normalisation come from the tensor cores too (the
// operand times a tile of ones, issued after the first block) and travel to
// the other CTAs on their own.  A split cluster barrier per step keeps a CTA
// from overwriting a receive buffer that another CTA is still reading.  The
// backward sweep reloads the resident slice with P's other orientation.  The
// per-step reference m_t comes from a small kernel that finds each weight's
// nearest codeword.
#include <cuda_runtime.h>

#include <cfloat>
#include <cmath>
#include <cstdint>

#include "bcjr_device.cuh"
#include "dense_internal.h"
#include "tc_util.cuh"

namespace bcjr {
namespace dtc {

using namespace tc;

constexpr int kS = kDenseStates;            // 256 states
constexpr int kCL = kDenseTCCluster;        // 4 CTAs per cluster = K-slices
constexpr int kSlice = kS / kCL;            // 64 states per CTA
constexpr int kKC = kSlice / 8;             // 8 K-chunks of 8 states
constexpr int kMR = kDenseTCRows;           // 128 sequences per cluster tile (MMA M)
constexpr int kWorkers = 256;              // 8 warps: two per tensor-memory lane quadrant
constexpr int kThreads = kWorkers + 32;     // + one warp that issues the MMAs
constexpr int kGroups = kSlice / 4;         // 16 groups of 4 states in a row's block
constexpr uint32_t kBTile = kS * 8 * 4;     // [256 rows][8 k] tf32 tile: 8 KiB
constexpr uint32_t kBBytes = kKC * 2 * kBTile;        // 8 K-chunks x (head, tail): 128 KiB
constexpr uint32_t kBBlock = 64 / 8 * 256;            // byte offset of the next 64 output rows in a tile
constexpr uint32_t kRxData = kMR * kSlice * 4;        // one sender's block: [16 groups][128 rows] float4, 32 KiB
constexpr uint32_t kRxSlot = kRxData + kMR * 4;       // + the sender's row sums [128]
constexpr uint32_t kRxBytes = (kCL - 1) * kRxSlot;    // bytes received per exchange
constexpr uint32_t kOnesBytes = 16 * 8 * 4;        // [16 rows][8 k] tile of ones: row sums on the tensor cores
constexpr uint32_t kOffB = 0, kOffRx = kBBytes, kOffOnes = kOffRx + kRxBytes;
constexpr uint32_t kOffCw = kOffOnes + kOnesBytes;   // this CTA's 64 codewords
constexpr uint32_t kOffBar = kOffCw + kSlice * 4;
constexpr uint32_t kSmemBytes = kOffBar + 96;
static_assert(kSmemBytes <= 227u * 1024u, "shared memory");
// Tensor memory: accumulator in columns [0, 256), operand head [256, 320) and
// tail [320, 384), the operand's row sums over this CTA's states in [384, 400).
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTAh = kS, kTAl = kS + kSlice, kTSum = kS + 2 * kSlice;
constexpr uint32_t kIdescN64 = idesc_tf32(64), kIdescN16 = idesc_tf32(16);

// Bulk copy global -> this CTA's shared memory, completing `bytes` on `bar`.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}

}  // namespace dtc

// The transfer matrix as resident slices: slice r of the forward image holds,
// for output state n and input state k in [64r, 64r+64), P[k][n]; slice r of
// the backward image holds P[n][k] (the product with P^T).  Each slice is
// [K-chunk c][head, tail][256 rows n][8 k] in K-major core-matrix tiles.
__global__ void dense_tc_prep_kernel(const float* __restrict__ lam, float* __restrict__ Bfwd,
                                     float* __restrict__ Bbwd, float* __restrict__ Prow) {
  using namespace dtc;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= kS * kS) return;
  const int row = i / kS, col = i - row * kS;
  const float pv = expf(lam[i]);  // P[row][col]
  if (Prow) Prow[i] = pv;
  float hi, lo;
  split_tf32(pv, hi, lo);
  auto put = [&](float* B, int nn, int kk) {
    const int r = kk / kSlice, c = (kk % kSlice) / 8, kc = (kk & 7) >> 2, e = kk & 3;
    unsigned char* base = reinterpret_cast<unsigned char*>(B) + static_cast<size_t>(r) * kBBytes + c * 2 * kBTile;
    const uint32_t off = chunk_off(nn, kc) + 4u * e;
    *reinterpret_cast<float*>(base + off) = hi;
    *reinterpret_cast<float*>(base + kBTile + off) = lo;
  };
  put(Bfwd, col, row);  // forward: output state col, input state row
  put(Bbwd, row, col);  // backward: output state row, input state col
}

// Reference of every (sequence, step): m = max_s -(w - c(s))^2 log2(e)/T, the
// value at the codeword nearest to w, computed with the same float operations
// as the emissions so that every factor 2^(phi - m) is at most one.
__global__ void dense_tc_mtab_kernel(const float* __restrict__ w, const float* __restrict__ codebook, float sc2,
                                     long long total, float* __restrict__ mtab) {
  using namespace dtc;
  __shared__ float cs[kS];
  const int tid = threadIdx.x;  // blockDim.x == kS
  const float ci = codebook[tid];
  int rank = 0;
  for (int j = 0; j < kS; ++j) {
    const float cj = codebook[j];
    rank += (cj < ci) || (cj == ci && j < tid);
  }
  cs[rank & (kS - 1)] = ci;
  __syncthreads();
  for (long long i = static_cast<long long>(blockIdx.x) * kS + tid; i < total; i += static_cast<long long>(gridDim.x) * kS) {
    const float wv = w[i];
    int lo = 0, hi = kS;  // first index with cs[idx] >= wv
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (cs[mid] < wv) {
        lo = mid + 1;
      } else {
        hi = mid;
      }
    }
    float best = -FLT_MAX;
    if (lo < kS) {
      const float d = wv - cs[lo];
      best = fmaxf(best, -(d * d) * sc2);
    }
    if (lo > 0) {
      const float d = wv - cs[lo - 1];
      best = fmaxf(best, -(d * d) * sc2);
    }
    mtab[i] = best;
  }
}

// ADJ: the vector-Jacobian product instead of the soft codeword; ROWS (with
// ADJ): also write the rows of the log-transition gradient.
template <bool ADJ, bool ROWS>
__global__ void __cluster_dims__(kDenseTCCluster, 1, 1) __launch_bounds__(dtc::kThreads, 1)
    dense_tc_kernel(const DenseTCParams p) {
  using namespace dtc;
  extern __shared__ __align__(16) unsigned char sm[];
  unsigned char* Bs = sm + kOffB;
  unsigned char* Rx = sm + kOffRx;
  float* ones = reinterpret_cast<float*>(sm + kOffOnes);
  const float* cws = reinterpret_cast<const float*>(sm + kOffCw);
  uint64_t* bar_c = reinterpret_cast<uint64_t*>(sm + kOffBar);  // [4] output blocks committed, in issue order
  uint64_t* bar_rx = bar_c + 4;                                  // [3] a receive slot filled
  uint64_t* bar_b = bar_c + 7;                                   // resident slice loaded
  uint64_t* bar_sum = bar_c + 8;                                 // row-sum MMAs done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_c + 9);
  int* abort_flag = reinterpret_cast<int*>(bar_c + 10);

  const int tid = threadIdx.x, warp = tid >> 5;
  const int r = static_cast<int>(cluster_rank());
  const int cid = static_cast<int>(blockIdx.x) / kCL, ncl = static_cast<int>(gridDim.x) / kCL;
  // Worker thread (half, row): states 32 half .. 32 half + 31 of every
  // 64-state block of row `row`, which is tensor-memory lane `row`.  Warp 8
  // issues the MMAs.
  const bool worker = tid < kWorkers;
  const int half = (warp >> 2) & 1;
  const int row = (warp & 3) * 32 + (tid & 31);
  const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
  const int n = p.n, N = p.N;
  constexpr int kSeqs = ADJ ? kMR / 2 : kMR;  // sequences per tile
  const int ntiles = (N + kSeqs - 1) / kSeqs;
  const float sc2 = p.sc2;

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid == 0) {
    for (int i = 0; i < 9; ++i) mbar_init(bar_c + i, 1);
    *abort_flag = 0;
    mbar_init_fence();
  }
  if (tid < kOnesBytes / 4) ones[tid] = 1.f;
  async_proxy_fence();  // the ones tile is read by the tensor cores
  if (tid < kSlice) reinterpret_cast<float*>(sm + kOffCw)[tid] = __ldg(p.codebook + r * kSlice + tid);
  const float* cw = cws + 32 * half;  // codewords of this thread's states
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (tid == 0)
    for (int i = 0; i < kCL - 1; ++i) mbar_arm(bar_rx + i, kRxSlot);
  cluster_sync_all();  // every CTA's barriers are initialised (and armed) before any remote store

  uint32_t ph_c[4] = {0, 0, 0, 0}, ph_b = 0, ph_sum = 0;
  uint32_t ph_rx = 0;  // parity of receive slot s in bit s
  // After one wait of this CTA gave up, no thread waits again (the call's results are void).
  auto waitb = [&](uint64_t* bar, uint32_t& ph) {
    if (!*reinterpret_cast<volatile int*>(abort_flag) && !mbar_wait(bar, ph, p.status, kDevTimeout))
      *reinterpret_cast<volatile int*>(abort_flag) = 1;
    ph ^= 1u;
  };

  // Load a resident slice (thread 0), completing on bar_b.
  auto load_b = [&](const float* image) {
    if (tid == 0) {
      mbar_arm(bar_b, kBBytes);
      const unsigned char* src = reinterpret_cast<const unsigned char*>(image) + static_cast<size_t>(r) * kBBytes;
#pragma unroll 1
      for (int q = 0; q < 8; ++q)
        bulk_g2s(smem_u32(Bs) + q * (kBBytes / 8), src + q * (kBBytes / 8), kBBytes / 8, smem_u32(bar_b));
    }
  };
  // Output block of issue slot k: the other CTAs' blocks first, the own one last.
  auto block_of = [&](int k) { return (r + 1 + k) & (kCL - 1); };
  // The MMAs of one step (one thread), one commit per output block; the
  // operand's row sums over this CTA's states (head and tail times a tile of
  // ones) follow the first block, so that the exchange starts as early as it
  // can.
  auto issue_mma = [&](bool first_of_sweep) {
    if (first_of_sweep) waitb(bar_b, ph_b);
    tc_fence_after();
    const bool go = !*reinterpret_cast<volatile int*>(abort_flag);
    const uint32_t b0 = smem_u32(Bs);
#pragma unroll 1
    for (int k = 0; k < kCL; ++k) {
      const int blk = block_of(k);
      const uint32_t d = tmem + static_cast<uint32_t>(blk * kSlice);
      if (go) {
#pragma unroll
        for (int c = 0; c < kKC; ++c) {
          const uint32_t bh = b0 + (2 * c) * kBTile + blk * kBBlock, bl = bh + kBTile;
          const uint32_t ah = tmem + kTAh + 8 * c, al = tmem + kTAl + 8 * c;
          mma_tf32_ts(d, ah, smem_desc(bh), kIdescN64, c > 0 ? 1u : 0u);  // hi * hi
          mma_tf32_ts(d, ah, smem_desc(bl), kIdescN64, 1u);               // hi * lo
          mma_tf32_ts(d, al, smem_desc(bh), kIdescN64, 1u);               // lo * hi
        }
      }
      mma_commit(bar_c + k);
      if (k == 0) {
        if (go) {
          const uint64_t od = smem_desc(smem_u32(ones));
#pragma unroll
          for (int c = 0; c < kKC; ++c) {
            mma_tf32_ts(tmem + kTSum, tmem + kTAh + 8 * c, od, kIdescN16, c > 0 ? 1u : 0u);
            mma_tf32_ts(tmem + kTSum, tmem + kTAl + 8 * c, od, kIdescN16, 1u);
          }
        }
        mma_commit(bar_sum);
      }
    }
  };
  // One step's contraction and reduce-scatter.  Every thread sends its half of
  // the other CTAs' blocks of its row as they complete (st.async into the
  // receiver's slot: 16 groups x 128 rows of float4, so a warp's stores are
  // contiguous; after the first block, half 0 sends the row sum to all three),
  // then adds the three received halves to its own into y.  Returns the row's sum of the consumed vector over all
  // 256 states, added in CTA order so that every CTA gets the same value.
  auto step = [&](bool first_of_sweep, float (&y)[32]) -> float {
    tc_fence_before();
    __syncthreads();  // operand written, accumulator read: the MMAs may go
    cluster_wait_plain();  // every CTA has read its receive buffer of the previous exchange
    float rs = 0.f;        // this CTA's part of the row sum
#pragma unroll 1
    for (int k = 0; k < kCL - 1; ++k) {
      const int blk = block_of(k);
      waitb(bar_c + k, ph_c[k]);
      tc_fence_after();
      uint32_t v[32];
      tmem_ld32_async(tmem + lane_off + static_cast<uint32_t>(blk * kSlice + 32 * half), v);
      tmem_wait_ld();
      const uint32_t slot = static_cast<uint32_t>(r < blk ? r : r - 1);
      const uint32_t dst = mapa_u32(smem_u32(Rx) + slot * kRxSlot, static_cast<uint32_t>(blk));
      const uint32_t rbar = mapa_u32(smem_u32(bar_rx + slot), static_cast<uint32_t>(blk));
#pragma unroll
      for (int g = 0; g < 8; ++g)
        st_async_v4f32(dst + static_cast<uint32_t>(((8 * half + g) * kMR + row) * 16), __uint_as_float(v[4 * g]),
                       __uint_as_float(v[4 * g + 1]), __uint_as_float(v[4 * g + 2]), __uint_as_float(v[4 * g + 3]),
                       rbar);
      if (k == 0) {
        waitb(bar_sum, ph_sum);
        tc_fence_after();
        uint32_t s1;
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(s1) : "r"(tmem + lane_off + kTSum));
        tmem_wait_ld();
        rs = __uint_as_float(s1);
        if (half == 0) {
#pragma unroll
          for (int j = 1; j < kCL; ++j) {
            const int b2 = (r + j) & (kCL - 1);
            const uint32_t sl2 = static_cast<uint32_t>(r < b2 ? r : r - 1);
            st_async_f32(mapa_u32(smem_u32(Rx) + sl2 * kRxSlot + kRxData + static_cast<uint32_t>(row * 4),
                                  static_cast<uint32_t>(b2)),
                         rs, mapa_u32(smem_u32(bar_rx + sl2), static_cast<uint32_t>(b2)));
          }
        }
      }
    }
    // Received halves: added as they land, in the order the senders finish
    // them (CTA r - 1 computes this CTA's block first); the own block's
    // partial sums come from the last commit.
#pragma unroll
    for (int j = 0; j < 32; ++j) y[j] = 0.f;
#pragma unroll 1
    for (int i = 0; i < kCL - 1; ++i) {
      if (i == kCL - 2) {
        waitb(bar_c + kCL - 1, ph_c[kCL - 1]);  // the last commit: every MMA of the step is done
        tc_fence_after();
        uint32_t v[32];
        tmem_ld32_async(tmem + lane_off + static_cast<uint32_t>(r * kSlice + 32 * half), v);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) y[j] += __uint_as_float(v[j]);
        tc_fence_before();
      }
      const int src = (r + kCL - 1 - i) & (kCL - 1);
      const int sl = src < r ? src : src - 1;
      uint32_t ph = (ph_rx >> sl) & 1u;
      waitb(bar_rx + sl, ph);
      ph_rx ^= 1u << sl;
      if (tid == 0) mbar_arm(bar_rx + sl, kRxSlot);  // the next exchange's phase
      const unsigned char* slot = Rx + sl * kRxSlot;
#pragma unroll
      for (int g = 0; g < 8; ++g) {
        const float4 q4 = *reinterpret_cast<const float4*>(slot + ((8 * half + g) * kMR + row) * 16);
        y[4 * g] += q4.x;
        y[4 * g + 1] += q4.y;
        y[4 * g + 2] += q4.z;
        y[4 * g + 3] += q4.w;
      }
    }
    float s = 0.f;
#pragma unroll
    for (int src = 0; src < kCL; ++src)
      s += src == r ? rs : *reinterpret_cast<const float*>(Rx + (src < r ? src : src - 1) * kRxSlot + kRxData + row * 4);
    cluster_arrive_relaxed();  // this CTA's receive buffer is read
    return s;
  };
  // The issuing warp's part of a sweep: the n - 1 steps' barriers and MMAs.
  auto issuer_sweep = [&]() {
    for (int t = 1; t < n; ++t) {
      tc_fence_before();
      __syncthreads();  // pairs with the workers' operand barrier
      if ((tid & 31) == 0) issue_mma(t == 1);
      __syncwarp();
      cluster_wait_plain();
      cluster_arrive_relaxed();
    }
  };
  // The next MMA's operand A: this thread's 32 values as tf32 head and tail.
  auto put_operand = [&](const float (&v)[32]) {
    uint32_t h[32], l[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      float fh, fl;
      split_tf32_int(v[j], fh, fl);
      h[j] = __float_as_uint(fh);
      l[j] = __float_as_uint(fl);
    }
    tmem_st32(tmem + lane_off + kTAh + 32 * half, h);
    tmem_st32(tmem + lane_off + kTAl + 32 * half, l);
    tmem_wait_st();
  };

  float gcacc[16];  // vector-Jacobian product: this thread's codebook-gradient sums
#pragma unroll
  for (int j = 0; j < 16; ++j) gcacc[j] = 0.f;
  float* ckbase = p.ck + static_cast<size_t>(cid * kCL + r) * p.ck_stride;      // [t][16 groups][128 rows] float4
  // [t][half][128 rows][2] partial sums, then [128 rows][half] the last forward row sums
  float* ptbase = p.part + static_cast<size_t>(cid * kCL + r) * p.part_stride;
  auto ck_at = [&](int t, int g) {
    return ckbase + ((static_cast<size_t>(t) * kGroups + 8 * half + g) * kMR + row) * 4;
  };

  for (int tile = cid; tile < ntiles; tile += ncl) {
    if constexpr (!ADJ) {
    const int q = tile * kMR + row;
    const bool act = q < N;
    const size_t qb = static_cast<size_t>(act ? q : 0) * n;  // padding rows run sequence 0 (discarded)

    // ---------------- forward sweep ----------------
    if (n > 1) load_b(p.Bfwd);  // one step has no contraction
    cluster_arrive_relaxed();   // pairs with the first step's wait
    double lsc = 0.0;           // log2 Z of the row: the references and log2 of the row sums
    if (!worker) issuer_sweep();
    float wn = __ldg(p.w + qb), mn = __ldg(p.mtab + qb);  // the step's weight and reference, loaded a step ahead
    float ps = 0.f;                                       // this thread's part of the current vector's row sum
    for (int t = 0; t < n && worker; ++t) {
      float y[32];
      float sprev = 1.f;
      if (t > 0) sprev = step(t == 1, y);
      const float wt = wn, mt = mn;
      if (t + 1 < n) {
        wn = __ldg(p.w + qb + t + 1);
        mn = __ldg(p.mtab + qb + t + 1);
      }
      const float inv = 1.f / sprev;
      ps = 0.f;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const float d = wt - cw[j];
        const float e = ex2f(-(d * d) * sc2 - mt);
        y[j] = (t > 0 ? y[j] * inv : 1.f) * e;
        ps += y[j];
      }
      lsc += static_cast<double>(mt) + (t > 0 ? static_cast<double>(log2f(sprev)) : 0.0);
#pragma unroll
      for (int g = 0; g < 8; ++g)
        *reinterpret_cast<float4*>(ck_at(t, g)) = make_float4(y[4 * g], y[4 * g + 1], y[4 * g + 2], y[4 * g + 3]);
      if (t + 1 < n) put_operand(y);
    }
    // For log Z: the last vector's row sum, by CTA and half, in the row after the partial sums.
    if (worker) ptbase[static_cast<size_t>(n) * 4 * kMR + row * 2 + half] = ps;
    cluster_wait_plain();  // pairs with the last arrive
    cluster_sync_all();    // every CTA is done with the forward sweep's exchanges

    // ---------------- backward sweep ----------------
    if (n > 1) load_b(p.Bbwd);
    cluster_arrive_relaxed();
    if (!worker) issuer_sweep();
    wn = __ldg(p.w + qb + n - 1);
    mn = __ldg(p.mtab + qb + n - 1);
    for (int t = n - 1; t >= 0 && worker; --t) {
      float z[32];
      float4 x4[8];  // the stored forward vector of the step, requested before the exchange
#pragma unroll
      for (int g = 0; g < 8; ++g) x4[g] = *reinterpret_cast<const float4*>(ck_at(t, g));
      float sig = 1.f;
      if (t < n - 1) sig = step(t == n - 2, z);
      const float wt = wn, mt = mn;
      if (t >= 1) {
        wn = __ldg(p.w + qb + t - 1);
        mn = __ldg(p.mtab + qb + t - 1);
      }
      const float inv = 1.f / sig;
      float den = 0.f, num = 0.f;
#pragma unroll
      for (int g = 0; g < 8; ++g) {
        const float xs[4] = {x4[g].x, x4[g].y, x4[g].z, x4[g].w};
        float gm[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j = 4 * g + e;
          z[j] = t < n - 1 ? z[j] * inv : 1.f;
          gm[e] = xs[e] * z[j];
          den += gm[e];
          num = fmaf(gm[e], cw[j], num);
        }
        if (p.marginals && act)
          *reinterpret_cast<float4*>(p.marginals + (static_cast<size_t>(q) * n + t) * kS + r * kSlice + 32 * half + 4 * g) =
              make_float4(gm[0], gm[1], gm[2], gm[3]);
      }
      // Partial sums over this thread's 32 states: (sum c gamma, sum gamma), by half.
      *reinterpret_cast<float2*>(ptbase + ((static_cast<size_t>(t) * 2 + half) * kMR + row) * 2) = make_float2(num, den);
      if (t >= 1) {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float d = wt - cw[j];
          z[j] = ex2f(-(d * d) * sc2 - mt) * z[j];
        }
        put_operand(z);
      }
    }
    cluster_wait_plain();
    cluster_sync_all();  // every CTA's partial sums (and marginal rows) are written

    // log Z (CTA 0, half 0): the forward references and row sums, and the last row sum over all states.
    if (r == 0 && worker && half == 0 && act) {
      float s = 0.f;
#pragma unroll
      for (int src = 0; src < kCL; ++src)
#pragma unroll
        for (int h = 0; h < 2; ++h)
          s += __ldcg(p.part + static_cast<size_t>(cid * kCL + src) * p.part_stride + static_cast<size_t>(n) * 4 * kMR +
                      row * 2 + h);
      const float lz = static_cast<float>((lsc + static_cast<double>(log2f(s))) * 0.69314718055994530942);
      if (!isfinite(lz)) atomicOr(p.status, kDevNonFinite);
      if (p.log_z) p.log_z[q] = lz;
    }
    // Soft codeword: CTA r takes the steps t = r, r + 4, ...; the partial sums
    // over the 8 state blocks are added in a fixed order.
    for (int t = r + kCL * (tid >> 7); t < n && worker; t += 2 * kCL) {
      const int rr = tid & (kMR - 1);
      const int qq = tile * kMR + rr;
      if (qq >= N) continue;
      float num = 0.f, den = 0.f;
#pragma unroll
      for (int src = 0; src < kCL; ++src)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          // other CTAs wrote these (at addresses earlier tiles also used): read through L2
          const float2 v = __ldcg(reinterpret_cast<const float2*>(
              p.part + static_cast<size_t>(cid * kCL + src) * p.part_stride + ((static_cast<size_t>(t) * 2 + h) * kMR + rr) * 2));
          num += v.x;
          den += v.y;
        }
      p.w_hat[static_cast<size_t>(qq) * n + t] = num / den;
    }
    // Marginals: this CTA's 64 states of every step, divided by the step's sum.
    if (p.marginals && worker) {
      for (int t = tid >> 7; t < n; t += 2) {
        const int rr = tid & (kMR - 1);
        const int qq = tile * kMR + rr;
        if (qq >= N) continue;
        float den = 0.f;
#pragma unroll
        for (int src = 0; src < kCL; ++src)
#pragma unroll
          for (int h = 0; h < 2; ++h)
            den += __ldcg(p.part + static_cast<size_t>(cid * kCL + src) * p.part_stride +
                          ((static_cast<size_t>(t) * 2 + h) * kMR + rr) * 2 + 1);
        const float inv = 1.f / den;
        float* mr = p.marginals + (static_cast<size_t>(qq) * n + t) * kS + r * kSlice;
#pragma unroll 4
        for (int j = 0; j < kSlice; j += 4) {
          float4 m4 = *reinterpret_cast<float4*>(mr + j);
          m4.x *= inv;
          m4.y *= inv;
          m4.z *= inv;
          m4.w *= inv;
          *reinterpret_cast<float4*>(mr + j) = m4;
        }
      }
    }
    cluster_sync_all();  // partial sums read before the next tile rewrites them
    } else {
      // ------------- vector-Jacobian product: 64 sequences, two operands each -------------
      // Row 2i + o of the MMA is operand o of sequence i of the tile: o = 0
      // carries the vector (x forward, v backward), o = 1 the vector times
      // its centred accumulator.  After a step the pair (2i, 2i + 1) trades
      // halves so that each thread holds both sums for 16 states: thread o
      // of the pair takes states c0 .. c0 + 15 of the CTA's block.
      const int o = row & 1, qi = row >> 1;
      const int ho = 2 * half + o;
      const int c0 = 32 * half + 16 * o;
      const int q = tile * kSeqs + qi;
      const bool act = q < N;
      const size_t qb = static_cast<size_t>(act ? q : 0) * n;  // padding sequences run sequence 0 (discarded)
      float* ckx = p.ck + static_cast<size_t>(cid * kCL + r) * p.ck_stride;
      float* ckf = p.ckf + static_cast<size_t>(cid * kCL + r) * p.ck_stride;
      float* cks = p.cks + static_cast<size_t>(cid * kCL + r) * p.cks_stride;
      // [t][pair half ho][float4 j][64 sequences] float4: a warp's stores are contiguous
      auto ck_off = [&](int t, int j) { return ((static_cast<size_t>(t) * 4 + ho) * 4 + j) * (kSeqs * 4) + qi * 4; };
      // per-row partial sums: [t][ho][64] for t < n, then [n][ho][64] last row sums, [n + 1][ho][64] D numerators
      auto part_at = [&](float* base, int t) { return base + (static_cast<size_t>(t) * 4 + ho) * kSeqs + qi; };
      // y (this thread's 32 sums of its row) -> a, b: the two operands' sums for states c0 .. c0 + 15
      auto pair_split = [&](const float (&y)[32], float (&a)[16], float (&b)[16]) {
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float other = __shfl_xor_sync(0xffffffffu, o == 0 ? y[16 + j] : y[j], 1);
          a[j] = o == 0 ? y[j] : other;
          b[j] = o == 0 ? other : y[16 + j];
        }
      };
      // the pair's operand rows from the two 16-state pieces of each thread
      auto put_pair = [&](const float (&v1)[16], const float (&v2)[16]) {
        float v[32];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float other = __shfl_xor_sync(0xffffffffu, o == 0 ? v2[j] : v1[j], 1);
          v[j] = o == 0 ? v1[j] : other;
          v[16 + j] = o == 0 ? other : v2[j];
        }
        put_operand(v);
      };
      const float* cwq = cws + c0;

      // ---------------- forward sweep: x_t and F~_t ----------------
      if (n > 1) load_b(p.Bfwd);
      cluster_arrive_relaxed();
      if (!worker) issuer_sweep();
      float wn = __ldg(p.w + qb), mn = __ldg(p.mtab + qb), gn = __ldg(p.g + qb), hn = __ldg(p.what_in + qb);
      float xsum = 0.f, dnum = 0.f;  // over this thread's states: the vector and its D numerator
      for (int t = 0; t < n && worker; ++t) {
        float y[32], a[16], b[16];
        float sprev = 1.f;
        if (t > 0) {
          const float s = step(t == 1, y);
          sprev = __shfl_sync(0xffffffffu, s, (threadIdx.x & 31) & ~1);  // the pair's vector row sum
          pair_split(y, a, b);
          if (half == 0 && o == 0) cks[static_cast<size_t>(t - 1) * kSeqs + qi] = sprev;  // s_{t-1}
        }
        const float wt = wn, mt = mn, gt = gn, ht = hn;
        if (t + 1 < n) {
          wn = __ldg(p.w + qb + t + 1);
          mn = __ldg(p.mtab + qb + t + 1);
          gn = __ldg(p.g + qb + t + 1);
          hn = __ldg(p.what_in + qb + t + 1);
        }
        const float inv = 1.f / sprev;
        float x[16], f[16], x2[16];
        xsum = 0.f;
        dnum = 0.f;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float c = cwq[j];
          const float d = wt - c;
          const float e = ex2f(-(d * d) * sc2 - mt);
          x[j] = (t > 0 ? a[j] * inv : 1.f) * e;
          f[j] = (t > 0 && a[j] > 0.f) ? __fdividef(b[j], a[j]) : 0.f;
          x2[j] = x[j] * (f[j] + gt * (c - ht));
          xsum += x[j];
          dnum += x2[j];
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          *reinterpret_cast<float4*>(ckx + ck_off(t, j)) = make_float4(x[4 * j], x[4 * j + 1], x[4 * j + 2], x[4 * j + 3]);
          *reinterpret_cast<float4*>(ckf + ck_off(t, j)) = make_float4(f[4 * j], f[4 * j + 1], f[4 * j + 2], f[4 * j + 3]);
        }
        if (t + 1 < n) put_pair(x, x2);
      }
      if (worker) {
        *part_at(ptbase, n) = xsum;  // last vector's row sum, and D's numerator, over this thread's states
        *part_at(ptbase, n + 1) = dnum;
      }
      cluster_wait_plain();
      cluster_sync_all();  // every CTA's partial sums of the last step are written

      // The last row sum s_{n-1} over all states (= den_{n-1}: z_{n-1} = 1) and
      // D = sum_s gamma_{n-1}(s) (F~_{n-1}(s) + eps_{n-1}(s)), added in a fixed order.
      float slast = 0.f, dsum = 0.f;
#pragma unroll
      for (int src = 0; src < kCL; ++src)
#pragma unroll
        for (int h4 = 0; h4 < 4; ++h4) {
          const float* pb = p.part + static_cast<size_t>(cid * kCL + src) * p.part_stride;
          slast += __ldcg(pb + (static_cast<size_t>(n) * 4 + h4) * kSeqs + qi);
          dsum += __ldcg(pb + (static_cast<size_t>(n + 1) * 4 + h4) * kSeqs + qi);
        }
      const float Dv = dsum / slast;
      if (worker && r == 0 && ho == 0 && act && !(isfinite(slast) && isfinite(Dv) && slast > 0.f))
        atomicOr(p.status, kDevNonFinite);
      // gamma's normaliser den_t = sum_s x_t(s) z_t(s) follows from the two
      // recursions' row sums: den_{t-1} = den_t s_{t-1} / sigma_t (s: forward
      // sums, sigma: backward sums), the same value on every CTA.
      double den = static_cast<double>(slast);

      // ---------------- backward sweep: z_t, B~_t, psi_t ----------------
      if (n > 1) load_b(p.Bbwd);
      cluster_arrive_relaxed();
      if (!worker) issuer_sweep();
      wn = __ldg(p.w + qb + n - 1);
      mn = __ldg(p.mtab + qb + n - 1);
      gn = __ldg(p.g + qb + n - 1);
      hn = __ldg(p.what_in + qb + n - 1);
      for (int t = n - 1; t >= 0 && worker; --t) {
        float4 x4[4], f4[4];  // the stored forward values of the step, requested before the exchange
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          x4[j] = *reinterpret_cast<const float4*>(ckx + ck_off(t, j));
          f4[j] = *reinterpret_cast<const float4*>(ckf + ck_off(t, j));
        }
        const float st = t < n - 1 ? cks[static_cast<size_t>(t) * kSeqs + qi] : 1.f;
        float y[32], a[16], b[16];
        float sig = 1.f;
        if (t < n - 1) {
          const float s = step(t == n - 2, y);
          sig = __shfl_sync(0xffffffffu, s, (threadIdx.x & 31) & ~1);
          pair_split(y, a, b);
          den = den * static_cast<double>(st) / static_cast<double>(sig);
        }
        const float wt = wn, mt = mn, gt = gn, ht = hn;
        if (t >= 1) {
          wn = __ldg(p.w + qb + t - 1);
          mn = __ldg(p.mtab + qb + t - 1);
          gn = __ldg(p.g + qb + t - 1);
          hn = __ldg(p.what_in + qb + t - 1);
        }
        const float inv = 1.f / sig;
        const float rden = static_cast<float>(1.0 / den);
        const float gsc = act ? gt : 0.f, tsc = act ? p.two_over_T : 0.f;
        // Rows of the log-transition gradient: X_t = x_t / n, U_t = x_t (F~ + eps - D) / n
        // for the transition t -> t + 1, with n = sum_p x_t(p) (P v_{t+1})(p) = sigma_{t+1} den_t;
        // V, W of the transition t - 1 -> t are the next operand's two rows.
        constexpr bool rows = ROWS;
        const float rn = act ? static_cast<float>(1.0 / (static_cast<double>(sig) * den)) : 0.f;
        const float ract = act ? 1.f : 0.f;
        const size_t rbase = static_cast<size_t>(cid) * p.row_region + static_cast<size_t>(r * kSlice + c0);
        float gw = 0.f;
        float v1[16], v2[16];
        float rx4[4], ru4[4];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float xs = (j & 3) == 0 ? x4[j >> 2].x : (j & 3) == 1 ? x4[j >> 2].y : (j & 3) == 2 ? x4[j >> 2].z : x4[j >> 2].w;
          const float fs = (j & 3) == 0 ? f4[j >> 2].x : (j & 3) == 1 ? f4[j >> 2].y : (j & 3) == 2 ? f4[j >> 2].z : f4[j >> 2].w;
          const float c = cwq[j];
          const float z = t < n - 1 ? a[j] * inv : 1.f;
          const float bt = (t < n - 1 && a[j] > 0.f) ? __fdividef(b[j], a[j]) : 0.f;
          const float eps = gt * (c - ht);
          const float gam = xs * z * rden;
          const float psi = gam * (fs + eps + bt - Dv);
          gw = fmaf(psi, c, gw);
          gcacc[j] += fmaf(gsc, gam, tsc * psi * (wt - c));
          const float d = wt - c;
          v1[j] = ex2f(-(d * d) * sc2 - mt) * z;
          v2[j] = v1[j] * (eps + bt);
          if (rows && t < n - 1) {
            rx4[j & 3] = xs * rn;
            ru4[j & 3] = xs * (fs + eps - Dv) * rn;
            if ((j & 3) == 3) {
              const size_t o = rbase + (static_cast<size_t>(t) * kSeqs + qi) * kS + (j & ~3);
              *reinterpret_cast<float4*>(p.rowX + o) = make_float4(rx4[0], rx4[1], rx4[2], rx4[3]);
              *reinterpret_cast<float4*>(p.rowU + o) = make_float4(ru4[0], ru4[1], ru4[2], ru4[3]);
            }
          }
        }
        if (rows && t >= 1) {
          const size_t o = rbase + (static_cast<size_t>(t - 1) * kSeqs + qi) * kS;
#pragma unroll
          for (int j = 0; j < 16; j += 4) {
            *reinterpret_cast<float4*>(p.rowV + o + j) =
                make_float4(ract * v1[j], ract * v1[j + 1], ract * v1[j + 2], ract * v1[j + 3]);
            *reinterpret_cast<float4*>(p.rowW + o + j) =
                make_float4(ract * v2[j], ract * v2[j + 1], ract * v2[j + 2], ract * v2[j + 3]);
          }
        }
        *part_at(ptbase, t) = gw;
        if (t >= 1) put_pair(v1, v2);
      }
      cluster_wait_plain();
      cluster_sync_all();  // every CTA's partial sums are written

      // grad_w: CTA r takes the steps t = r, r + 4, ...; the partial sums over
      // 4 CTAs x 4 pieces of 16 states are added in a fixed order.
      for (int t = r + kCL * (tid >> 6); t < n && worker; t += 4 * kCL) {
        const int qq = tid & (kSeqs - 1);
        const int qg = tile * kSeqs + qq;
        if (qg >= N) continue;
        float gw = 0.f;
#pragma unroll
        for (int src = 0; src < kCL; ++src)
#pragma unroll
          for (int h4 = 0; h4 < 4; ++h4)
            gw += __ldcg(p.part + static_cast<size_t>(cid * kCL + src) * p.part_stride +
                         (static_cast<size_t>(t) * 4 + h4) * kSeqs + qq);
        p.grad_w[static_cast<size_t>(qg) * n + t] = p.two_over_T * gw;
      }
      cluster_sync_all();  // partial sums read before the next tile rewrites them
    }
  }

  if constexpr (ADJ) {
    // This CTA's 64 codebook-gradient sums: over the 16 sequences of a warp
    // with equal pair side (lane shuffles), then over the 4 lane quadrants
    // (the receive area is free now), in a fixed order.
    float* red = reinterpret_cast<float*>(Rx);  // [4 quadrants][64 states]
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      float v = gcacc[j];
#pragma unroll
      for (int off = 2; off < 32; off <<= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
      gcacc[j] = v;
    }
    if (worker && (tid & 31) < 2) {
      const int c0 = 32 * half + 16 * (tid & 1);
#pragma unroll
      for (int j = 0; j < 16; ++j) red[(warp & 3) * kSlice + c0 + j] = gcacc[j];
    }
    __syncthreads();
    if (tid < kSlice)
      p.gc_part[static_cast<size_t>(cid) * kS + r * kSlice + tid] =
          ((red[tid] + red[kSlice + tid]) + red[2 * kSlice + tid]) + red[3 * kSlice + tid];
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
  cluster_sync_all();  // no CTA leaves while its shared memory may be addressed
}

// ---------------------------------------------------------------------------
// Host side.
// ---------------------------------------------------------------------------
size_t dense_tc_smem_bytes() { return dtc::kSmemBytes; }

namespace {
// Per device and variant: the kernel's shared-memory attribute is set and its
// cluster occupancy queried once, so that later calls issue no driver queries
// (a query can wait behind other users of the driver).  0 = not yet known.
constexpr int kMaxDevices = 64;
int g_tc_clusters[3][kMaxDevices] = {};

template <bool ADJ, bool ROWS>
int tc_clusters_of_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 0;
  if (dev < kMaxDevices && g_tc_clusters[ADJ + ROWS][dev] > 0) return g_tc_clusters[ADJ + ROWS][dev];
  const size_t smem = dense_tc_smem_bytes();
  if (cudaFuncSetAttribute(dense_tc_kernel<ADJ, ROWS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return 0;
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(dtc::kCL * sms, 1, 1);
  cfg.blockDim = dim3(dtc::kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  int clusters = 0;
  if (cudaOccupancyMaxActiveClusters(&clusters, dense_tc_kernel<ADJ, ROWS>, &cfg) != cudaSuccess) return 0;
  if (dev < kMaxDevices) g_tc_clusters[ADJ + ROWS][dev] = clusters;
  return clusters;
}
}  // namespace

int dense_tc_max_clusters(bool adjoint) {
  // the row-writing variant has the same resources as the plain adjoint
  return adjoint ? tc_clusters_of_device<true, false>() : tc_clusters_of_device<false, false>();
}

cudaError_t launch_dense_tc(const DenseTCParams& p, const float* lam, bool adjoint, int clusters, cudaStream_t s) {
  using namespace dtc;
  dense_tc_prep_kernel<<<(kS * kS + 255) / 256, 256, 0, s>>>(lam, p.Bfwd, p.Bbwd, p.P);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const long long total = static_cast<long long>(p.N) * p.n;
  const long long blocks = (total + kS - 1) / kS;
  dense_tc_mtab_kernel<<<static_cast<unsigned>(blocks < 4096 ? blocks : 4096), kS, 0, s>>>(p.w, p.codebook, p.sc2, total,
                                                                                         p.mtab);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // the occupancy queries also set the kernels' shared-memory attribute
  const bool rows = adjoint && p.rowX != nullptr;
  if (rows) {
    if (tc_clusters_of_device<true, true>() < 1) return cudaErrorNotSupported;
    dense_tc_kernel<true, true><<<clusters * kCL, kThreads, dense_tc_smem_bytes(), s>>>(p);
  } else if (adjoint) {
    if (tc_clusters_of_device<true, false>() < 1) return cudaErrorNotSupported;
    dense_tc_kernel<true, false><<<clusters * kCL, kThreads, dense_tc_smem_bytes(), s>>>(p);
  } else {
    if (tc_clusters_of_device<false, false>() < 1) return cudaErrorNotSupported;
    dense_tc_kernel<false, false><<<clusters * kCL, kThreads, dense_tc_smem_bytes(), s>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace bcjr
