// xu_probe.cu -- throughput of the special-function (XU) pipe: the measured
// peak behind the exp-pipe roofline of the forward-backward kernels.
//
// One CTA of 1024 threads per SM keeps 32 warps resident; every thread runs 16
// independent chains of dependent ex2 (or lg2) instructions, so the pipe, not
// the latency of one chain, sets the pace.  Each CTA counts its own cycles.
#include <cuda_runtime.h>

#include "bcjr.h"
#include "bcjr_probe.h"

namespace {

constexpr int kProbeThreads = 1024;
constexpr int kChains = 16;

template <int OP>
__global__ void __launch_bounds__(kProbeThreads, 1) xu_probe_kernel(int iters, float* __restrict__ sink,
                                                                    long long* __restrict__ cycles) {
  float v[kChains];
#pragma unroll
  for (int i = 0; i < kChains; ++i) v[i] = 0.25f + 0.03125f * static_cast<float>(i) + 1e-6f * threadIdx.x;
  __syncthreads();
  const long long t0 = clock64();
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int i = 0; i < kChains; ++i) {
      if constexpr (OP == 0) {
        // v <- 2^(-v): stays in (0.5, 1) for v in (0, 1)
        asm volatile("{\n\t.reg .f32 t;\n\tneg.f32 t, %1;\n\tex2.approx.ftz.f32 %0, t;\n\t}" : "=f"(v[i]) : "f"(v[i]));
      } else {
        // v <- log2(v + 3): stays in (1.58, 2.33) for v in (0, 2.33)
        asm volatile("{\n\t.reg .f32 t;\n\tadd.f32 t, %1, 0f40400000;\n\tlg2.approx.ftz.f32 %0, t;\n\t}"
                     : "=f"(v[i])
                     : "f"(v[i]));
      }
    }
  }
  __syncthreads();
  const long long t1 = clock64();
  if (threadIdx.x == 0) cycles[blockIdx.x] = t1 - t0;
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < kChains; ++i) s += v[i];
  sink[static_cast<size_t>(blockIdx.x) * kProbeThreads + threadIdx.x] = s;
}

}  // namespace

extern "C" bcjr_status bcjr_probe_xu(int op, int iters, float* sink, long long* cycles, int n_sm,
                                     bcjr_stream_t stream) {
  if ((op != BCJR_PROBE_EX2 && op != BCJR_PROBE_LG2) || iters < 1 || iters > (1 << 20) || !sink || !cycles ||
      n_sm < 1 || n_sm > 4096)
    return BCJR_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (op == BCJR_PROBE_EX2) {
    xu_probe_kernel<0><<<n_sm, kProbeThreads, 0, s>>>(iters, sink, cycles);
  } else {
    xu_probe_kernel<1><<<n_sm, kProbeThreads, 0, s>>>(iters, sink, cycles);
  }
  return cudaGetLastError() == cudaSuccess ? BCJR_OK : BCJR_ERR_CUDA;
}
