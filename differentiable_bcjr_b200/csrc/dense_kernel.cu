// dense_kernel.cu -- vector-Jacobian product over a dense (fully connected)
// trellis that also writes the rows of the log-transition gradient (sm_100a):
// the kernel behind bcjr_dense_backward_lambda.  The soft codeword and the
// plain vector-Jacobian product run on the tensor cores (dense_tc_kernel.cu);
// this kernel keeps all 256 states of a sequence in one CTA so that it can
// write the full-width rows X, U, V, W that dense_dlam_kernel.cu sums.
//
// "BCJR-QAT: A Differentiable Relaxation of Trellis-Coded Weight Quantization",
// abstract: the relaxation is a 1D Ising-like chain solved by a transfer
// matrix.  With log-transition Lambda[p][s] (row = source state) and emission
// phi_t(s) = -(w_t - c(s))^2 / T, the path weight is
//     exp(sum_t phi_t(s_t) + sum_{t>=1} Lambda[s_{t-1}][s_t]),  uniform start, free end.
//
// Probability domain, one normalisation per step (P = exp(Lambda)):
//   forward   x_0 = E_0,  x_t = (x_{t-1} P) (.) E_t,  E_t(s) = 2^{phi2_t(s) - max_s phi2_t},
//             each row rescaled by its sum (log2 of the scales summed for log Z);
//   backward  z_{n-1} = 1, z_{t-1} = (E_t (.) z_t) P^T, rescaled likewise;
//   gamma_t   = x_t (.) z_t / sum_s x_t z_t.
// Every recursion contracts (a dense chain forgets its start within a few
// steps), so float32 rounding does not accumulate along the sequence.
// The vector-Jacobian product uses the same centred accumulators as the
// bitshift kernels, now one dense contraction each:
//   F~_u = ((x_{u-1} (.) (F~_{u-1} + eps_{u-1})) P) / (x_{u-1} P),
//   B~_u = ((v_{u+1} (.) (eps_{u+1} + B~_{u+1})) P^T) / (v_{u+1} P^T),  v = E (.) z,
//   psi_u = gamma_u (.) (F~_u + eps_u + B~_u - D),  eps_u = g_u (c - w_hat_u),
// stacked as a second operand of the same contraction.
//
// Layout.  A CTA owns kM = 32 sequences (rows) and all 256 states (columns).
// Each step is one [32 x 256] x [256 x 256] contraction: the operand rows sit
// in shared memory (column-major, 16-byte slots XOR-swizzled so that both the
// row-broadcast reads and the transposing writes are conflict-free) and P or
// P^T streams through a double-buffered shared-memory window of 32 rows with
// cp.async.  A thread holds 4 sequences x 8 states (states 4l..4l+3 and
// 128+4l..128+4l+3 of lane l), 8 warps per CTA, so state sums are warp shuffles; the
// contraction runs on packed f32x2 fused multiply-adds over state pairs (each
// lane rounds exactly as a scalar fma would).
#include <cuda_runtime.h>

#include <cmath>

#include "bcjr_device.cuh"
#include "dense_internal.h"

namespace bcjr {
namespace dense {

constexpr int kS = kDenseStates;  // 256
constexpr int kM = kDenseRows;    // 32 sequences per CTA
constexpr int kKC = 32;           // rows of P per shared-memory window
constexpr int kChunks = kS / kKC;
constexpr float kLog2e = 1.4426950408889634f;

struct Cfg {
  static constexpr int RQ = 4;  // sequences per thread (8 warps per CTA)
  static constexpr int WARPS = kM / RQ;
  static constexpr int THREADS = 32 * WARPS;
};

// State held by slot j of lane l.
__device__ __forceinline__ int st_of(int lane, int j) { return j < 4 ? 4 * lane + j : 128 + 4 * lane + (j - 4); }

// Operand tile [S][M]: row s holds the 32 sequences as 8 slots of 4 floats;
// slot g of row s is stored at slot g ^ ((s >> 2) & 7).
__device__ __forceinline__ int a_index(int s, int q) {
  return s * kM + ((((q >> 2) ^ (s >> 2)) & 7) << 2) + (q & 3);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

}  // namespace dense

__global__ void dense_prep_kernel(const float* __restrict__ lam, float* __restrict__ P, float* __restrict__ PT,
                                  int S) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < S * S) {
    const int r = i / S, c = i - r * S;
    const float v = expf(lam[i]);
    P[i] = v;
    PT[static_cast<size_t>(c) * S + r] = v;
  }
}

__global__ void __launch_bounds__(dense::Cfg::THREADS, 1) dense_adj_kernel(const DenseParams p) {
  using namespace dense;
  constexpr int RQ = Cfg::RQ;
  constexpr int NTH = Cfg::THREADS;
  extern __shared__ __align__(16) float sm[];
  float* A1 = sm;                           // [S][M] first operand
  float* A2 = A1 + kS * kM;                 // [S][M] second operand (adjoint)
  float* Pc = A2 + kS * kM;     // [2][KC][S] window of P or P^T
  float* stX = Pc + 2 * kKC * kS;           // [M][S] staged x_t (backward)
  float* stF = stX + kM * kS;               // [M][S] staged F~_t (adjoint backward)

  const int tid = threadIdx.x, wp = tid >> 5, lane = tid & 31;
  const int n = p.n, N = p.N;
  const int nblk = (N + kM - 1) / kM;
  const float sc2 = p.sc2;

  float cs[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) cs[j] = __ldg(p.codebook + st_of(lane, j));
  float gcacc[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) gcacc[j] = 0.f;

  float* ckx = p.ckx + static_cast<size_t>(blockIdx.x) * p.ck_stride;
  float* ckf = p.ckf + static_cast<size_t>(blockIdx.x) * p.ck_stride;
  float* mtab = p.mtab + static_cast<size_t>(blockIdx.x) * p.mt_stride;

  // One 32-row window of B (P or P^T) into buffer `buf`, plus optional extra 16-byte copies.
  auto issue_window = [&](const float* B, int kc, int buf) {
    const float* src = B + static_cast<size_t>(kc) * kKC * kS;
    float* dst = Pc + buf * kKC * kS;
#pragma unroll
    for (int r = 0; r < (kKC * kS) / (4 * NTH); ++r) {
      const int i = (tid + r * NTH) * 4;
      cp_async16(dst + i, src + i);
    }
  };
  auto issue_stage = [&](int t) {  // x_t (and F~_t) of this CTA's rows into the staging tiles
    const float* srcx = ckx + static_cast<size_t>(t) * kM * kS;
    const float* srcf = ckf + static_cast<size_t>(t) * kM * kS;
#pragma unroll
    for (int r = 0; r < (kM * kS) / (4 * NTH); ++r) {
      const int i = (tid + r * NTH) * 4;
      cp_async16(stX + i, srcx + i);
      cp_async16(stF + i, srcf + i);
    }
  };

  // acc1 (acc2) = A1 (A2) x B.  Window 0 of B must already be in flight in
  // buffer 0; window 0 of `Bnext` is issued at the end, and `stage_t` >= 0
  // stages that step's checkpoint alongside window 1.
  auto contract = [&](const float* B, const float* Bnext, int stage_t, float (&acc1)[RQ][8], float (&acc2)[RQ][8]) {
#pragma unroll
    for (int i = 0; i < RQ; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        acc1[i][j] = 0.f;
        acc2[i][j] = 0.f;
      }
    for (int kc = 0; kc < kChunks; ++kc) {
      cp_async_wait<0>();
      __syncthreads();  // window kc landed; every thread is done with window kc-1 and wrote its operands
      if (kc + 1 < kChunks) issue_window(B, kc + 1, (kc + 1) & 1);
      if (kc == 0 && stage_t >= 0) issue_stage(stage_t);
      cp_async_commit();
      const float* Pb = Pc + (kc & 1) * kKC * kS;
#pragma unroll 8
      for (int kk = 0; kk < kKC; ++kk) {
        const int s = kc * kKC + kk;
        const float4 b0 = *reinterpret_cast<const float4*>(Pb + kk * kS + 4 * lane);
        const float4 b1 = *reinterpret_cast<const float4*>(Pb + kk * kS + 128 + 4 * lane);
        const float2 bv2[4] = {make_float2(b0.x, b0.y), make_float2(b0.z, b0.w), make_float2(b1.x, b1.y),
                               make_float2(b1.z, b1.w)};
#pragma unroll
        for (int g = 0; g < RQ / 4; ++g) {
          const int q = RQ * wp + 4 * g;
          const float4 a = *reinterpret_cast<const float4*>(A1 + a_index(s, q));
          const float av[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
          for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              float2 c2 = make_float2(acc1[4 * g + i][2 * j], acc1[4 * g + i][2 * j + 1]);
              c2 = __ffma2_rn(make_float2(av[i], av[i]), bv2[j], c2);
              acc1[4 * g + i][2 * j] = c2.x;
              acc1[4 * g + i][2 * j + 1] = c2.y;
            }
          {
            const float4 a2 = *reinterpret_cast<const float4*>(A2 + a_index(s, q));
            const float av2[4] = {a2.x, a2.y, a2.z, a2.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                float2 c2 = make_float2(acc2[4 * g + i][2 * j], acc2[4 * g + i][2 * j + 1]);
                c2 = __ffma2_rn(make_float2(av2[i], av2[i]), bv2[j], c2);
                acc2[4 * g + i][2 * j] = c2.x;
                acc2[4 * g + i][2 * j + 1] = c2.y;
              }
          }
        }
      }
    }
    cp_async_wait<0>();
    __syncthreads();  // every thread is done with both windows and the operands
    if (Bnext) {
      issue_window(Bnext, 0, 0);
      cp_async_commit();
    }
  };

  for (int blk = blockIdx.x; blk < nblk; blk += gridDim.x) {
    int qg[RQ];
    bool act[RQ];
#pragma unroll
    for (int i = 0; i < RQ; ++i) {
      qg[i] = blk * kM + RQ * wp + i;
      act[i] = qg[i] < N;
    }
    auto load_row = [&](const float* base, int i, int t) { return act[i] ? __ldg(base + static_cast<size_t>(qg[i]) * n + t) : 0.f; };

    float acc1[RQ][8], acc2[RQ][8];
    double lsc[RQ];
    float Dv[RQ];
#pragma unroll
    for (int i = 0; i < RQ; ++i) {
      lsc[i] = 0.0;
      Dv[i] = 0.f;
    }
    // ---------------- forward sweep ----------------
    if (n > 1) {
      issue_window(p.P, 0, 0);
      cp_async_commit();
    }
    for (int t = 0; t < n; ++t) {
      if (t > 0) contract(p.P, t + 1 < n ? p.P : p.PT, -1, acc1, acc2);
#pragma unroll
      for (int i = 0; i < RQ; ++i) {
        const int q = RQ * wp + i;
        const float wt = load_row(p.w, i, t);
        float ph[8];
        float mx = -INFINITY;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float d = wt - cs[j];
          ph[j] = -(d * d) * sc2;
          mx = fmaxf(mx, ph[j]);
        }
        const float m2 = warp_max(mx);
        float x[8], F[8];
        float sum = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float e = ex2f(ph[j] - m2);
          x[j] = (t > 0) ? acc1[i][j] * e : e;
          F[j] = (t > 0 && acc1[i][j] > 0.f) ? acc2[i][j] / acc1[i][j] : 0.f;
          sum += x[j];
        }
        const float sig = warp_sum(sum);
        const float inv = 1.f / sig;
        lsc[i] += static_cast<double>(m2) + static_cast<double>(log2f(sig));
        float eps[8];
        float gt = 0.f, wh = 0.f;
        {
          gt = load_row(p.g, i, t);
          wh = load_row(p.what_in, i, t);
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          x[j] *= inv;
          eps[j] = gt * (cs[j] - wh);
        }
        if (lane == 0) mtab[static_cast<size_t>(t) * kM + q] = m2;
        float* cx = ckx + (static_cast<size_t>(t) * kM + q) * kS;
        *reinterpret_cast<float4*>(cx + 4 * lane) = make_float4(x[0], x[1], x[2], x[3]);
        *reinterpret_cast<float4*>(cx + 128 + 4 * lane) = make_float4(x[4], x[5], x[6], x[7]);
        {
          float* cf = ckf + (static_cast<size_t>(t) * kM + q) * kS;
          *reinterpret_cast<float4*>(cf + 4 * lane) = make_float4(F[0], F[1], F[2], F[3]);
          *reinterpret_cast<float4*>(cf + 128 + 4 * lane) = make_float4(F[4], F[5], F[6], F[7]);
        }
        if (t + 1 < n) {
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            A1[a_index(st_of(lane, j), q)] = x[j];
            A2[a_index(st_of(lane, j), q)] = x[j] * (F[j] + eps[j]);
          }
        } else {
          // D = E[sum_u eps_u] = sum_s gamma_{n-1}(s) (F~_{n-1}(s) + eps_{n-1}(s)); z_{n-1} = 1
          float dsum = 0.f;
#pragma unroll
          for (int j = 0; j < 8; ++j) dsum = fmaf(x[j], F[j] + eps[j], dsum);
          Dv[i] = warp_sum(dsum);
        }
      }
    }
    if (lane == 0) {
#pragma unroll
      for (int i = 0; i < RQ; ++i)
        if (act[i] && !(isfinite(lsc[i]) && isfinite(Dv[i]))) atomicOr(p.status, kDevNonFinite);
    }

    // ---------------- backward sweep ----------------
    // stage x_{n-1} (and F~_{n-1}); every thread wrote its own rows, so a barrier orders them
    __syncthreads();
    issue_stage(n - 1);
    cp_async_commit();
    cp_async_wait<0>();
    __syncthreads();
    for (int t = n - 1; t >= 0; --t) {
#pragma unroll
      for (int i = 0; i < RQ; ++i) {
        const int q = RQ * wp + i;
        float x[8], z[8], Fv[8], Bt[8];
        {
          const float4 x0 = *reinterpret_cast<const float4*>(stX + q * kS + 4 * lane);
          const float4 x1 = *reinterpret_cast<const float4*>(stX + q * kS + 128 + 4 * lane);
          x[0] = x0.x; x[1] = x0.y; x[2] = x0.z; x[3] = x0.w;
          x[4] = x1.x; x[5] = x1.y; x[6] = x1.z; x[7] = x1.w;
          {
            const float4 f0 = *reinterpret_cast<const float4*>(stF + q * kS + 4 * lane);
            const float4 f1 = *reinterpret_cast<const float4*>(stF + q * kS + 128 + 4 * lane);
            Fv[0] = f0.x; Fv[1] = f0.y; Fv[2] = f0.z; Fv[3] = f0.w;
            Fv[4] = f1.x; Fv[5] = f1.y; Fv[6] = f1.z; Fv[7] = f1.w;
          }
        }
        float zsum = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          z[j] = (t < n - 1) ? acc1[i][j] : 1.f;
          Bt[j] = (t < n - 1 && acc1[i][j] > 0.f) ? acc2[i][j] / acc1[i][j] : 0.f;
          zsum += z[j];
        }
        const float zinv = 1.f / warp_sum(zsum);
        float gsum = 0.f;
        float gm[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          z[j] *= zinv;
          gm[j] = x[j] * z[j];
          gsum += gm[j];
        }
        const float den = warp_sum(gsum);
        const float ginv = 1.f / den;
        const float wt = load_row(p.w, i, t);
        float eps[8];
        {
          const float gt = load_row(p.g, i, t);
          const float wh = load_row(p.what_in, i, t);
          const float actf = act[i] ? 1.f : 0.f;
          float gw = 0.f;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            eps[j] = gt * (cs[j] - wh);
            const float g_ = gm[j] * ginv;
            const float psi = g_ * (Fv[j] + eps[j] + Bt[j] - Dv[i]);
            gw = fmaf(psi, cs[j], gw);
            gcacc[j] += actf * fmaf(gt, g_, p.two_over_T * psi * (wt - cs[j]));
          }
          gw = warp_sum(gw);
          if (act[i] && lane == 0) p.grad_w[static_cast<size_t>(qg[i]) * n + t] = p.two_over_T * gw;
          if (p.ckv && t < n - 1) {
            // Rows of the log-transition gradient for the transition t -> t+1:
            // X = x_t / n, U = x_t (F~_t + eps_t - D) / n with n = sum_s x_t(s) (P v_{t+1})(s)
            // = den / zinv.  They replace this step's checkpoint, already staged.
            const float sn = act[i] ? zinv * ginv : 0.f;
            float X8[8], U8[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              X8[j] = x[j] * sn;
              U8[j] = x[j] * (Fv[j] + eps[j] - Dv[i]) * sn;
            }
            float* xr = ckx + (static_cast<size_t>(t) * kM + q) * kS;
            float* ur = ckf + (static_cast<size_t>(t) * kM + q) * kS;
            *reinterpret_cast<float4*>(xr + 4 * lane) = make_float4(X8[0], X8[1], X8[2], X8[3]);
            *reinterpret_cast<float4*>(xr + 128 + 4 * lane) = make_float4(X8[4], X8[5], X8[6], X8[7]);
            *reinterpret_cast<float4*>(ur + 4 * lane) = make_float4(U8[0], U8[1], U8[2], U8[3]);
            *reinterpret_cast<float4*>(ur + 128 + 4 * lane) = make_float4(U8[4], U8[5], U8[6], U8[7]);
          }
        }
        if (t >= 1) {
          const float m2 = mtab[static_cast<size_t>(t) * kM + q];
          float V8[8], W8[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float d = wt - cs[j];
            const float v = ex2f(-(d * d) * sc2 - m2) * z[j];
            A1[a_index(st_of(lane, j), q)] = v;
            V8[j] = v;
            {
              W8[j] = v * (eps[j] + Bt[j]);
              A2[a_index(st_of(lane, j), q)] = W8[j];
            }
          }
          {
            if (p.ckv) {  // rows V = v_t, W = v_t (eps_t + B~_t) of the transition t-1 -> t
              float* vr = p.ckv + static_cast<size_t>(blockIdx.x) * p.ck_stride + (static_cast<size_t>(t - 1) * kM + q) * kS;
              float* wr = p.ckw + static_cast<size_t>(blockIdx.x) * p.ck_stride + (static_cast<size_t>(t - 1) * kM + q) * kS;
              *reinterpret_cast<float4*>(vr + 4 * lane) = make_float4(V8[0], V8[1], V8[2], V8[3]);
              *reinterpret_cast<float4*>(vr + 128 + 4 * lane) = make_float4(V8[4], V8[5], V8[6], V8[7]);
              *reinterpret_cast<float4*>(wr + 4 * lane) = make_float4(W8[0], W8[1], W8[2], W8[3]);
              *reinterpret_cast<float4*>(wr + 128 + 4 * lane) = make_float4(W8[4], W8[5], W8[6], W8[7]);
            }
          }
        }
      }
      if (t >= 1) contract(p.PT, t > 1 ? p.PT : nullptr, t - 1, acc1, acc2);
    }
  }

  {
    // Per-CTA codebook-gradient partial: sum the warps' per-lane accumulators in a fixed order.
    __syncthreads();
    float* red = Pc;  // [WARPS][S]
#pragma unroll
    for (int j = 0; j < 8; ++j) red[wp * kS + st_of(lane, j)] = gcacc[j];
    __syncthreads();
    for (int s = tid; s < kS; s += NTH) {
      float v = 0.f;
      for (int w = 0; w < Cfg::WARPS; ++w) v += red[w * kS + s];
      p.gc_part[static_cast<size_t>(blockIdx.x) * kS + s] = v;
    }
  }
}

// ---------------------------------------------------------------------------
// Host side.
// ---------------------------------------------------------------------------
size_t dense_smem_bytes() {
  using namespace dense;
  return sizeof(float) * (2 * kS * kM + 2 * kKC * kS + 2 * kM * kS);
}

int dense_max_grid() {
  const size_t smem = dense_smem_bytes();
  if (cudaFuncSetAttribute(dense_adj_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
      cudaSuccess)
    return 0;
  int dev = 0, sms = 0, per_sm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, dense_adj_kernel, dense::Cfg::THREADS, smem) != cudaSuccess)
    return 0;
  return per_sm * sms;
}

cudaError_t launch_dense_prep(const float* lam, const DenseParams& p, cudaStream_t s) {
  const int S = dense::kS;
  dense_prep_kernel<<<(S * S + 255) / 256, 256, 0, s>>>(lam, const_cast<float*>(p.P), const_cast<float*>(p.PT), S);
  return cudaGetLastError();
}

cudaError_t launch_dense(const DenseParams& p, const float* lam, int grid, cudaStream_t s, bool prep) {
  cudaError_t e = cudaSuccess;
  if (prep && (e = launch_dense_prep(lam, p, s)) != cudaSuccess) return e;
  dense_adj_kernel<<<grid, dense::Cfg::THREADS, dense_smem_bytes(), s>>>(p);
  return cudaGetLastError();
}

}  // namespace bcjr
