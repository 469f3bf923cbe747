// bcjr_device.cuh -- device-side building blocks of the bitshift-trellis kernels.
//
// Team geometry.  One weight sequence is processed by a "team" of S/16
// threads; every thread owns the same 16 trellis states for the whole launch,
// so its 16 codewords stay in registers and its 16 codebook-gradient
// accumulators never leave registers either.  A team is
//   * a thread-block cluster of CL CTAs when S/16 > 1024 (L = 15, 16),
//   * one CTA when 32 <= S/16 <= 1024,
//   * a slice of one warp (several teams per CTA) when S/16 < 32.
//
// Unit tiling.  With Q = S/K^2 "units" q, unit q holds the K x K states
//   s = (j << (L-k)) | (q << k) | b,      j, b in [0, K).
// For fixed b the K states (over j) share the predecessor group of
// g = (q << k) | b (the forward log-sum-exp); for fixed j the K states (over b)
// are the successors of every state p with p & (S/K-1) == (j << (L-2k)) | q
// (the backward log-sum-exp).  A thread holds a JT x BT tile of one unit
// (K >= 4) or U whole units (K = 2); when K >= 8 the K/4 x K/4 tiles of a unit
// sit in consecutive lanes and combine their partial sums with shuffles.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace bcjr {

constexpr int kStatesPerThread = 16;

constexpr int ilog2_constexpr(int v) { return v <= 1 ? 0 : 1 + ilog2_constexpr(v >> 1); }

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float lg2f(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float rcpf(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// The .aligned cluster barriers require every lane of the warp to execute
// them together; lanes that ran a divergent branch just before (e.g. lane 0
// publishing a warp result) are re-joined first, so that their stores precede
// the warp's arrival.
__device__ __forceinline__ void cluster_sync_all() {
  __syncwarp();
  asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
               "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Store v into the shared memory of CTA `rank` of this cluster at the same
// offset as the local address `p`.
__device__ __forceinline__ void st_cluster_f32(const float* p, uint32_t rank, float v) {
  uint32_t a = smem_u32(p), r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(r), "f"(v) : "memory");
}
__device__ __forceinline__ void st_cluster_v4(const float* p, uint32_t rank, float4 v) {
  uint32_t a = smem_u32(p), r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
  asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(r), "f"(v.x), "f"(v.y),
               "f"(v.z), "f"(v.w)
               : "memory");
}
__device__ __forceinline__ void st_cluster_f64(const double* p, uint32_t rank, double v) {
  uint32_t a = smem_u32(p), r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
  asm volatile("st.shared::cluster.f64 [%0], %1;" ::"r"(r), "d"(v) : "memory");
}
__device__ __forceinline__ void st_cluster_u32(const void* p, uint32_t rank, uint32_t v) {
  uint32_t a = smem_u32(p), r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(r), "r"(v) : "memory");
}

template <int CL>
__device__ __forceinline__ void team_store(float* base, uint32_t rank, int off, float v) {
  if constexpr (CL == 1) {
    base[off] = v;
  } else {
    st_cluster_f32(base + off, rank, v);
  }
}
template <int CL>
__device__ __forceinline__ void team_store_f64(double* base, uint32_t rank, int off, double v) {
  if constexpr (CL == 1) {
    base[off] = v;
  } else {
    st_cluster_f64(base + off, rank, v);
  }
}
template <int CL>
__device__ __forceinline__ void team_store_u32(uint32_t* base, uint32_t rank, int off, uint32_t v) {
  if constexpr (CL == 1) {
    base[off] = v;
  } else {
    st_cluster_u32(base + off, rank, v);
  }
}

template <int CL>
__device__ __forceinline__ void team_sync() {
  if constexpr (CL == 1) {
    __syncthreads();
  } else {
    cluster_sync_all();
  }
}

// Max over aligned groups of `width` lanes (width a power of two <= 32).
__device__ __forceinline__ float group_max(float v, int width) {
  if (width == 32) {
    float r;
    asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
    return r;
  }
  for (int o = width >> 1; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float group_sum(float v, int width) {
  for (int o = width >> 1; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ double group_sum_f64(double v, int width) {
  for (int o = width >> 1; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Compile-time tile shape for 2^k predecessors.
template <int K>
struct Tile {
  static constexpr int JT = K < 4 ? K : 4;                   // j values per thread
  static constexpr int BT = K < 4 ? K : 4;                   // b values per thread
  static constexpr int U = K <= 4 ? 16 / (K * K) : 1;        // whole units per thread
  static constexpr int TPU = K <= 4 ? 1 : (K * K) / 16;      // threads per unit
  static constexpr int NBT = K / BT;                         // b-tiles per unit
  static_assert(U * JT * BT == kStatesPerThread, "16 states per thread");
};

}  // namespace bcjr

namespace bcjr {

__device__ __forceinline__ void st_cluster_v2f64(const double* p, uint32_t rank, double a, double b) {
  uint32_t addr = smem_u32(p), r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  asm volatile("st.shared::cluster.v2.f64 [%0], {%1, %2};" ::"r"(r), "d"(a), "d"(b) : "memory");
}

// Split cluster barrier: arrive (release) now, wait (acquire) later.
__device__ __forceinline__ void cluster_arrive() {
  __syncwarp();
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  __syncwarp();
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Asynchronous 16-byte global -> shared copy, completed with cp_async_wait<N>.
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem)), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async4(void* smem, const void* gmem) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(smem)), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ double group_max_f64(double v, int width) {
  for (int o = width >> 1; o > 0; o >>= 1) v = fmax(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

}  // namespace bcjr

namespace bcjr {

// ---------------------------------------------------------------------------
// Asynchronous exchange between the CTAs of a cluster.  A value is written
// into another CTA's shared memory with st.async, which also counts its bytes
// against an mbarrier in that CTA; a reader waits on its own mbarrier until
// the bytes of the step have arrived.  No release fence is involved, so a
// writer never stalls on the completion of its own stores.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t mapa_u32(uint32_t local_addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local_addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
// Make initialised mbarriers visible to the other CTAs of the cluster.
__device__ __forceinline__ void mbar_init_fence() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
// One arrival that also announces `bytes` of incoming transactions for the current phase.
__device__ __forceinline__ void mbar_arm(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
// Bound of every device-side wait: about two seconds of SM clock.
constexpr long long kWaitLimitCycles = 4000000000LL;

// Wait for the phase with the given parity to complete (acquire at cluster
// scope, so the other CTAs' st.async data is visible).  Gives up after
// `limit` SM clock cycles, ORs `timeout_bit` into *status and returns false.
// One try: true once the phase with the given parity has completed.  The hint
// lets the thread sleep in hardware until the phase completes (or 0.1 ms
// pass) instead of re-issuing a loop.
__device__ __forceinline__ bool mbar_try(uint32_t a, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(a), "r"(parity), "r"(100000u)
      : "memory");
  return done != 0;
}
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int* status, int timeout_bit,
                                          long long limit = kWaitLimitCycles) {
  const uint32_t a = smem_u32(bar);
  if (mbar_try(a, parity)) return true;  // the usual case: no clock reads
  const long long t0 = clock64();
  while (true) {
    if (mbar_try(a, parity)) return true;
    if (clock64() - t0 > limit) {
      atomicOr(status, timeout_bit);
      return false;
    }
  }
}
// st.async of one or two float64, or of one, two or four float32, into cluster shared
// memory at `raddr`, completing their bytes on the mbarrier at `rbar` (both
// addresses already mapped to the destination CTA).
__device__ __forceinline__ void st_async_f64(uint32_t raddr, double v, uint32_t rbar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.f64 [%0], %1, [%2];" ::"r"(raddr), "d"(v),
               "r"(rbar)
               : "memory");
}
__device__ __forceinline__ void st_async_v2f64(uint32_t raddr, double a, double b, uint32_t rbar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.f64 [%0], {%1, %2}, [%3];" ::"r"(raddr),
               "d"(a), "d"(b), "r"(rbar)
               : "memory");
}
__device__ __forceinline__ void st_async_f32(uint32_t raddr, float v, uint32_t rbar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.f32 [%0], %1, [%2];" ::"r"(raddr), "f"(v),
               "r"(rbar)
               : "memory");
}
__device__ __forceinline__ void st_async_v2f32(uint32_t raddr, float a, float b, uint32_t rbar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.f32 [%0], {%1, %2}, [%3];" ::"r"(raddr),
               "f"(a), "f"(b), "r"(rbar)
               : "memory");
}
__device__ __forceinline__ void st_async_v4f32(uint32_t raddr, float a, float b, float c, float d, uint32_t rbar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.f32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(
                   raddr),
               "f"(a), "f"(b), "f"(c), "f"(d), "r"(rbar)
               : "memory");
}
// Bulk copy of `bytes` (a multiple of 16; both addresses 16-byte aligned) from
// this CTA's shared memory at `src` into cluster shared memory at `dst`,
// completing on the mbarrier at `rbar` (dst and rbar mapped to the destination
// CTA).  The source must stay unchanged until the destination's mbarrier
// phase has completed.
__device__ __forceinline__ void bulk_copy_s2c(uint32_t dst, uint32_t src, uint32_t bytes, uint32_t rbar) {
  asm volatile("cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   dst),
               "r"(src), "r"(bytes), "r"(rbar)
               : "memory");
}
// Orders this thread's generic-proxy shared-memory writes before later
// async-proxy operations (bulk copies, tensor-core reads) on them.
__device__ __forceinline__ void async_proxy_fence() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
// Split cluster barrier without memory ordering: it only orders the
// execution of the threads (every read of a buffer before its next overwrite).
__device__ __forceinline__ void cluster_arrive_relaxed() {
  __syncwarp();
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_plain() {
  __syncwarp();
  asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
}

}  // namespace bcjr
