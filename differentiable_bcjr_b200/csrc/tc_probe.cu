// tc_probe.cu -- measurement aids behind the dense trellis's tensor-core
// design and the clusters' exchange: the issue cost of one tf32 tensor-core
// product (tcgen05.mma with operand A in tensor memory) as a function of N,
// and the bandwidth of the distributed-shared-memory exchange between the
// CTAs of a 4-CTA cluster, moved by per-thread st.async stores or by bulk
// copies.  They are what bound a step of the dense kernels (the per-step
// reduce-scatter and the per-step MMAs), measured on the device at hand.
#include <cuda_runtime.h>

#include <cstdint>

#include "bcjr.h"
#include "bcjr_common.h"
#include "bcjr_device.cuh"
#include "bcjr_probe.h"
#include "tc_util.cuh"

namespace {

using namespace bcjr;
using namespace bcjr::tc;

constexpr int kMmaThreads = 128;
constexpr uint32_t kMmaSmem = 65536;  // B tile (up to [256][8] tf32 = 8 KiB) and spare room

// One CTA per SM: thread 0 issues `iters` products D[128 x N] (+)= A[128 x 8] B[8 x N]
// into tensor-memory columns [0, N), A read from columns [256, 264), B an
// [N][8] K-major tile in shared memory; one commit, one bounded wait.
template <int N>
__global__ void __launch_bounds__(kMmaThreads, 1) mma_probe_kernel(int iters, long long* __restrict__ cycles,
                                                                   int* __restrict__ status) {
  extern __shared__ __align__(1024) unsigned char sm[];
  __shared__ uint64_t bar;
  __shared__ uint32_t slot;
  const int tid = threadIdx.x;
  for (int i = tid; i < static_cast<int>(kMmaSmem / 4); i += kMmaThreads)
    reinterpret_cast<float*>(sm)[i] = 0.001f * static_cast<float>(i & 7);
  if (tid < 32) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(smem_u32(&slot))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid == 0) mbar_init(&bar, 1);
  async_proxy_fence();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = slot;
  if (tid == 0) {
    const uint64_t bd = smem_desc(smem_u32(sm));
    constexpr uint32_t idesc = idesc_tf32(N);
    const long long t0 = clock64();
    for (int i = 0; i < iters; ++i) mma_tf32_ts(tm, tm + 256u, bd, idesc, i > 0 ? 1u : 0u);
    mma_commit(&bar);
    mbar_wait(&bar, 0u, status, kDevTimeout);
    cycles[blockIdx.x] = clock64() - t0;
  }
  tc_fence_before();
  __syncthreads();
  if (tid < 32) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tm) : "memory");
  }
}

constexpr int kXThreads = 256;
constexpr uint32_t kXSlot = 32768;             // one sender's 32 KiB
constexpr uint32_t kXSmem = 3 * kXSlot + 64;   // three receive slots + the mbarrier

__device__ __forceinline__ void st_async_v4(uint32_t raddr, float4 v, uint32_t rbar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.f32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(
                   raddr),
               "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w), "r"(rbar)
               : "memory");
}

// 4-CTA clusters: per round every CTA stores `reps` x 32 KiB into each of its
// three peers' receive slots with st.async (a warp's 16-byte stores are 512
// contiguous bytes), and waits (bounded) for the 3 x reps x 32 KiB it receives.
__global__ void __cluster_dims__(4, 1, 1) __launch_bounds__(kXThreads, 1)
    dsmem_probe_kernel(int reps, int rounds, long long* __restrict__ cycles, int* __restrict__ status) {
  extern __shared__ __align__(1024) unsigned char sm[];
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + 3 * kXSlot);
  const uint32_t rank = cluster_rank();
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    mbar_init_fence();
  }
  __syncthreads();
  cluster_sync_all();
  const uint32_t total = 3u * kXSlot * static_cast<uint32_t>(reps);
  const float4 v = make_float4(1.f, 2.f, 3.f, static_cast<float>(threadIdx.x));
  bool timed_out = false;
  const long long t0 = clock64();
  for (int it = 0; it < rounds; ++it) {
    if (threadIdx.x == 0) mbar_arm(bar, total);
    cluster_arrive_relaxed();  // every CTA has armed before any data of the round lands
    cluster_wait_plain();
    for (int rep = 0; rep < reps; ++rep)
      for (uint32_t j = 1; j < 4; ++j) {
        const uint32_t peer = (rank + j) & 3u;
        const uint32_t sl = rank < peer ? rank : rank - 1;
        const uint32_t dst = mapa_u32(smem_u32(sm) + sl * kXSlot, peer);
        const uint32_t rb = mapa_u32(smem_u32(bar), peer);
#pragma unroll
        for (int g = 0; g < 8; ++g) st_async_v4(dst + 16u * (g * kXThreads + threadIdx.x), v, rb);
      }
    if (!timed_out) timed_out = !mbar_wait(bar, static_cast<uint32_t>(it & 1), status, kDevTimeout);
  }
  const long long t1 = clock64();
  if (threadIdx.x == 0) cycles[blockIdx.x] = t1 - t0;
  cluster_sync_all();  // no CTA leaves while its shared memory may be addressed
}

constexpr uint32_t kXSmemBulk = 4 * kXSlot + 64;  // three receive slots, one source slot, the mbarrier

// The same exchange as dsmem_probe_kernel, moved by the bulk-copy engine: each
// warp owns 4 KiB of every 32 KiB slot and its lanes issue one
// cp.async.bulk (shared::cta -> shared::cluster, completing on the receiver's
// mbarrier) per `chunk` bytes of it, from a local source slot written once.
__global__ void __cluster_dims__(4, 1, 1) __launch_bounds__(kXThreads, 1)
    dsmem_bulk_probe_kernel(int chunk, int reps, int rounds, long long* __restrict__ cycles, int* __restrict__ status) {
  extern __shared__ __align__(1024) unsigned char sm[];
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + 4 * kXSlot);
  float4* src = reinterpret_cast<float4*>(sm + 3 * kXSlot);
  const uint32_t rank = cluster_rank();
  for (int i = threadIdx.x; i < static_cast<int>(kXSlot / 16); i += kXThreads)
    src[i] = make_float4(1.f, 2.f, 3.f, static_cast<float>(i));
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    mbar_init_fence();
  }
  async_proxy_fence();  // the source's generic-proxy writes before the copies read it
  __syncthreads();
  cluster_sync_all();
  constexpr uint32_t kPerWarp = kXSlot / (kXThreads / 32);
  const uint32_t ch = static_cast<uint32_t>(chunk);
  const uint32_t nch = kPerWarp / ch;
  const uint32_t warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t total = 3u * kXSlot * static_cast<uint32_t>(reps);
  const uint32_t src_base = smem_u32(src) + warp * kPerWarp;
  bool timed_out = false;
  const long long t0 = clock64();
  for (int it = 0; it < rounds; ++it) {
    if (threadIdx.x == 0) mbar_arm(bar, total);
    cluster_arrive_relaxed();
    cluster_wait_plain();
    for (int rep = 0; rep < reps; ++rep)
      for (uint32_t i = lane; i < 3u * nch; i += 32u) {
        const uint32_t peer = (rank + 1u + i / nch) & 3u;
        const uint32_t c = i % nch;
        const uint32_t sl = rank < peer ? rank : rank - 1;
        const uint32_t dst = mapa_u32(smem_u32(sm) + sl * kXSlot + warp * kPerWarp + c * ch, peer);
        bulk_copy_s2c(dst, src_base + c * ch, ch, mapa_u32(smem_u32(bar), peer));
      }
    if (!timed_out) timed_out = !mbar_wait(bar, static_cast<uint32_t>(it & 1), status, kDevTimeout);
  }
  const long long t1 = clock64();
  if (threadIdx.x == 0) cycles[blockIdx.x] = t1 - t0;
  cluster_sync_all();
}

}  // namespace

extern "C" bcjr_status bcjr_probe_mma_tf32(int n, int iters, long long* cycles, int* status, int n_sm,
                                           bcjr_stream_t stream) {
  if (iters < 1 || iters > (1 << 20) || !cycles || !status || n_sm < 1 || n_sm > 4096) return BCJR_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaSuccess;
  switch (n) {
#define BCJR_MMA_PROBE_CASE(NN)                                                                                 \
  case NN:                                                                                                     \
    e = cudaFuncSetAttribute(mma_probe_kernel<NN>, cudaFuncAttributeMaxDynamicSharedMemorySize, kMmaSmem);     \
    if (e == cudaSuccess) mma_probe_kernel<NN><<<n_sm, kMmaThreads, kMmaSmem, s>>>(iters, cycles, status);     \
    break;
    BCJR_MMA_PROBE_CASE(16)
    BCJR_MMA_PROBE_CASE(32)
    BCJR_MMA_PROBE_CASE(64)
    BCJR_MMA_PROBE_CASE(128)
    BCJR_MMA_PROBE_CASE(256)
#undef BCJR_MMA_PROBE_CASE
    default:
      return BCJR_ERR_INVALID_ARG;
  }
  if (e == cudaSuccess) e = cudaGetLastError();
  return e == cudaSuccess ? BCJR_OK : BCJR_ERR_CUDA;
}

extern "C" bcjr_status bcjr_probe_dsmem(int reps, int rounds, long long* cycles, int* status, int n_clusters,
                                        bcjr_stream_t stream) {
  if (reps < 1 || reps > 8 || rounds < 1 || rounds > (1 << 16) || !cycles || !status || n_clusters < 1 ||
      n_clusters > 1024)
    return BCJR_ERR_INVALID_ARG;
  cudaError_t e = cudaFuncSetAttribute(dsmem_probe_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kXSmem);
  if (e == cudaSuccess) {
    dsmem_probe_kernel<<<4 * n_clusters, kXThreads, kXSmem, reinterpret_cast<cudaStream_t>(stream)>>>(
        reps, rounds, cycles, status);
    e = cudaGetLastError();
  }
  return e == cudaSuccess ? BCJR_OK : BCJR_ERR_CUDA;
}

extern "C" bcjr_status bcjr_probe_dsmem_bulk(int chunk_bytes, int reps, int rounds, long long* cycles, int* status,
                                             int n_clusters, bcjr_stream_t stream) {
  const bool chunk_ok = chunk_bytes >= 128 && chunk_bytes <= 4096 && (chunk_bytes & (chunk_bytes - 1)) == 0;
  if (!chunk_ok || reps < 1 || reps > 8 || rounds < 1 || rounds > (1 << 16) || !cycles || !status ||
      n_clusters < 1 || n_clusters > 1024)
    return BCJR_ERR_INVALID_ARG;
  cudaError_t e =
      cudaFuncSetAttribute(dsmem_bulk_probe_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kXSmemBulk);
  if (e == cudaSuccess) {
    dsmem_bulk_probe_kernel<<<4 * n_clusters, kXThreads, kXSmemBulk, reinterpret_cast<cudaStream_t>(stream)>>>(
        chunk_bytes, reps, rounds, cycles, status);
    e = cudaGetLastError();
  }
  return e == cudaSuccess ? BCJR_OK : BCJR_ERR_CUDA;
}
