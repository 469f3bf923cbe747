// dense_dlam_kernel.cu -- gradient with respect to the log-transitions of the
// dense trellis, accumulated on the fifth-generation tensor cores (sm_100a).
//
// "BCJR-QAT: A Differentiable Relaxation of Trellis-Coded Weight Quantization",
// technical summary, "key technical innovations": the soft codeword is exactly
// differentiable in the trellis parameters; abstract: the dense chain is a
// transfer-matrix (1D Ising-like) computation.  Lambda[p][r] enters the path
// log-weight once per transition p -> r, so with G = sum_u g_u c(s_u),
//     dL/dLambda[p][r] = Cov(G, #transitions p -> r)
//                      = sum_{seq, u >= 1} xi_u(p, r) (a_{u-1}(p) + b_u(r) - D),
// xi_u the pairwise posterior of (s_{u-1}, s_u), a the past and b the future
// part of the centred loss (the accumulators F~ and B~ of the adjoint sweep).
// In the probability domain xi_u(p, r) = P[p][r] x_{u-1}(p) v_u(r) / n_u, so
//     dL/dLambda = P (.) sum_rows (X^T W + U^T V),
//     X = x / n,  U = x (a - D) / n,  V = v,  W = v b,
// where the backward (adjoint) kernel writes one row of X, U, V, W per
// (sequence, transition).  This kernel is that sum: a [256 x R] x [R x 256]
// contraction over R = (sequences x transitions) rows, split over the CTAs.
//
// Tensor cores.  Each CTA owns the full 256 x 256 float32 accumulator in
// tensor memory (two M = 128 halves side by side: all 512 columns).  Rows
// stream through shared memory eight at a time (one tf32 MMA step of K = 8):
// the CTA's threads load them with coalesced loads, split every value into a
// tf32 head and a tail (x = hi + lo, hi rounded to tf32, lo exact in float32)
// and store both into K-major, non-swizzled core-matrix tiles; one thread then
// issues, per M half, the three products hi*hi + hi*lo + lo*hi of each operand
// pair (3xTF32: the dropped lo*lo term is ~2^-22 relative, where a single tf32
// product would leave ~5e-4 relative error in the sum), and commits them to an
// mbarrier that frees the stage buffer.  Two stage buffers let the loads and
// splits of one stage overlap the MMAs of the other.  At the end the threads
// read the accumulator back with tcgen05.ld and write the CTA's partial sum;
// a reduction kernel adds the partials in a fixed order and applies P (.).
#include <cuda_runtime.h>

#include <cstdint>

#include "bcjr_device.cuh"
#include "dense_internal.h"
#include "tc_util.cuh"

namespace bcjr {
namespace dlam {
using namespace tc;

constexpr int kS = kDenseStates;                    // 256
constexpr int kK = 8;                               // rows per stage (one tf32 MMA step)
constexpr int kThreads = 256;
constexpr uint32_t kTileBytes = kS * kK * 4;         // 8 KiB: [256][8] tf32 operand tile
constexpr int kTiles = 8;                           // X hi/lo, U hi/lo, W hi/lo, V hi/lo
constexpr uint32_t kStageBytes = kTiles * kTileBytes;  // 64 KiB
constexpr int kStages = 2;
constexpr uint32_t kTmemCols = 512;                 // 2 x (M = 128 lanes, N = 256 columns) float32

}  // namespace dlam

// One CTA per SM (the accumulator takes all of the SM's tensor memory).
// Stages [s0, s1) of the R / 8 row stages; stage s covers rows 8 s .. 8 s + 7
// of region s / spr (spr stages per region; a region is one backward CTA's
// rows, `region_stride` floats apart).
__global__ void __launch_bounds__(dlam::kThreads, 1) dense_dlam_kernel(const DlamParams p) {
  using namespace dlam;
  extern __shared__ __align__(1024) unsigned char dl_smem[];
  // Stage buffers on a 1 KiB boundary; bookkeeping after them.
  const uint32_t raw = smem_u32(dl_smem);
  const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
  unsigned char* stage_base = dl_smem + pad;
  uint64_t* bar_free = reinterpret_cast<uint64_t*>(stage_base + kStages * kStageBytes);  // [kStages]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_free + kStages);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long total = p.total_stages;
  const long long s0 = total * blockIdx.x / gridDim.x, s1 = total * (blockIdx.x + 1) / gridDim.x;

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid == 0) {
    for (int b = 0; b < kStages; ++b) mbar_init(bar_free + b, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // This thread's column (state) of every row.
  const int col = tid;
  const float* srcs[4] = {p.X, p.U, p.W, p.V};  // tile pairs: (X, W) and (U, V)
  float cur[4][kK];
  auto load_stage = [&](long long s) {
    const long long region = s / p.spr;
    const long long row0 = (s - region * p.spr) * kK;
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const float* src = srcs[m] + region * p.region_stride + row0 * kS + col;
#pragma unroll
      for (int k = 0; k < kK; ++k) cur[m][k] = __ldg(src + k * kS);
    }
  };

  bool timed_out = false;
  bool first = true;
  if (s0 < s1) load_stage(s0);
  for (long long s = s0; s < s1; ++s) {
    // Stage i uses buffer i & 1 for the (i >> 1)-th time; the MMAs of its
    // previous use must be complete before the buffer is rewritten.
    const long long i = s - s0;
    const int b = static_cast<int>(i & 1);
    if (i >= 2 && !timed_out)
      timed_out = !mbar_wait(bar_free + b, static_cast<uint32_t>(((i >> 1) - 1) & 1), p.status, kDevTimeout);
    unsigned char* buf = stage_base + b * kStageBytes;
    // Tiles: 0 X hi, 1 X lo, 2 U hi, 3 U lo, 4 W hi, 5 W lo, 6 V hi, 7 V lo.
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const int t_hi = m == 0 ? 0 : m == 1 ? 2 : m == 2 ? 4 : 6;
#pragma unroll
      for (int kc = 0; kc < 2; ++kc) {
        float h[4], l[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) split_tf32(cur[m][4 * kc + e], h[e], l[e]);
        const uint32_t off = chunk_off(col, kc);
        *reinterpret_cast<float4*>(buf + t_hi * kTileBytes + off) = make_float4(h[0], h[1], h[2], h[3]);
        *reinterpret_cast<float4*>(buf + (t_hi + 1) * kTileBytes + off) = make_float4(l[0], l[1], l[2], l[3]);
      }
    }
    if (s + 1 < s1) load_stage(s + 1);  // the next stage's loads overlap this stage's MMAs
    async_proxy_fence();                // generic-proxy stores -> visible to the tensor core
    __syncthreads();
    if (tid == 0 && !timed_out) {
      tc_fence_after();
      const uint32_t base = smem_u32(buf);
#pragma unroll
      for (int h = 0; h < 2; ++h) {  // M halves: rows 0..127 and 128..255 of the accumulator
        const uint32_t d = tmem + static_cast<uint32_t>(h * kS);
        const uint32_t ah = static_cast<uint32_t>(h) * (kTileBytes / 2);  // 16 row groups of 256 B
#pragma unroll
        for (int pr = 0; pr < 2; ++pr) {  // (X, W) then (U, V)
          const uint32_t A = base + (pr == 0 ? 0u : 2u) * kTileBytes + ah;
          const uint32_t B = base + (pr == 0 ? 4u : 6u) * kTileBytes;
          mma_tf32(d, smem_desc(A), smem_desc(B), (first && pr == 0) ? 0u : 1u);     // hi * hi
          mma_tf32(d, smem_desc(A), smem_desc(B + kTileBytes), 1u);                  // hi * lo
          mma_tf32(d, smem_desc(A + kTileBytes), smem_desc(B), 1u);                  // lo * hi
        }
      }
      mma_commit(bar_free + b);
    }
    first = false;
  }
  // Wait for the last commit of each buffer: then every MMA has completed.
  const long long cnt = s1 - s0;
  for (int b = 0; b < kStages; ++b) {
    const long long uses = (cnt - b + 1) / 2;  // stages that used buffer b
    if (uses > 0 && !timed_out)
      timed_out = !mbar_wait(bar_free + b, static_cast<uint32_t>((uses - 1) & 1), p.status, kDevTimeout);
  }
  // Every thread waited on its own; the accumulator is read only if none gave up.
  const bool have = (s0 < s1) && !__syncthreads_or(timed_out);
  tc_fence_after();

  // Epilogue: warps 0-3 read accumulator half 0 (rows 0..127), warps 4-7 half 1.
  {
    const int half = warp >> 2, quad = warp & 3;
    const int row = half * 128 + quad * 32 + lane;
    float* dst = p.part + static_cast<size_t>(blockIdx.x) * kS * kS + static_cast<size_t>(row) * kS;
#pragma unroll 1
    for (int c = 0; c < kS / 32; ++c) {
      float v[32];
      if (have) {
        tmem_ld32(tmem + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(half * kS + c * 32), v);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = 0.f;
      }
#pragma unroll
      for (int i = 0; i < 32; i += 4)
        *reinterpret_cast<float4*>(dst + c * 32 + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

// out = (accumulate ? out : 0) + P (.) sum_c part[c], the partials in a fixed order.
__global__ void dense_dlam_reduce_kernel(const float* __restrict__ part, int nparts, const float* __restrict__ P,
                                         float* __restrict__ out, int accumulate) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  constexpr int kSS = kDenseStates * kDenseStates;
  if (i >= kSS) return;
  float s = 0.f;
  for (int c = 0; c < nparts; ++c) s += part[static_cast<size_t>(c) * kSS + i];
  const float v = P[i] * s;
  out[i] = accumulate ? out[i] + v : v;
}

size_t dlam_smem_bytes() { return 1024 + dlam::kStages * dlam::kStageBytes + 64; }

cudaError_t dlam_grid(long long total_stages, int* grid) {
  const size_t smem = dlam_smem_bytes();
  cudaError_t e =
      cudaFuncSetAttribute(dense_dlam_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  long long g = total_stages < sms ? total_stages : sms;
  *grid = static_cast<int>(g < 1 ? 1 : g);
  return cudaSuccess;
}

cudaError_t launch_dlam(const DlamParams& p, int grid, cudaStream_t s) {
  if (p.total_stages > 0) {
    dense_dlam_kernel<<<grid, dlam::kThreads, dlam_smem_bytes(), s>>>(p);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_dlam_reduce(const float* part, int nparts, const float* P, float* out, int accumulate,
                               cudaStream_t s) {
  constexpr int kSS = kDenseStates * kDenseStates;
  dense_dlam_reduce_kernel<<<kSS / 256, 256, 0, s>>>(part, nparts, P, out, accumulate);
  return cudaGetLastError();
}

}  // namespace bcjr
