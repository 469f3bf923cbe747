// dense_internal.h -- launch parameters of the dense (fully connected) trellis
// kernels, shared by the C-ABI layer and the kernels.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "bcjr_common.h"

namespace bcjr {

// Dense (fully connected) trellis: 256 states, 32 sequences per CTA.
constexpr int kDenseStates = 256;
constexpr int kDenseRows = 32;

struct DenseParams {
  const float* w;          // [N][n]
  const float* codebook;   // [S]
  const float* g;          // [N][n] upstream gradient (backward)
  const float* what_in;    // [N][n] soft codeword of the forward call (backward; centring)
  float* w_hat;            // [N][n] (forward)
  float* marginals;        // [N][n][S] or null (forward)
  float* log_z;            // [N] or null (forward)
  float* grad_w;           // [N][n] (backward)
  float* gc_part;          // [grid][S] per-CTA codebook-gradient partials (backward)
  const float* P;          // [S][S] exp(Lambda)
  const float* PT;         // [S][S] its transpose
  float* ckx;              // per CTA [n][32][S] normalised forward vectors
  float* ckf;              // per CTA [n][32][S] forward adjoint accumulators (backward)
  float* ckv;              // per CTA [n][32][S] rows V of the log-transition gradient, or null
  float* ckw;              // per CTA [n][32][S] rows W of the log-transition gradient (with ckv)
  float* mtab;             // per CTA [n][32] emission reference of each step
  int* status;
  size_t ck_stride;        // floats per CTA in ckx / ckf
  size_t mt_stride;        // floats per CTA in mtab
  float sc2;               // log2(e) / T
  float two_over_T;
  int n, N;
};

// Soft codeword of the dense trellis on the tensor cores (dense_tc_kernel.cu):
// a cluster of kDenseTCCluster CTAs per kDenseTCRows sequences, CTA r holding
// K-slice r of the transfer matrix.
constexpr int kDenseTCCluster = 4;
constexpr int kDenseTCRows = 128;

struct DenseTCParams {
  const float* w;          // [N][n]
  const float* codebook;   // [S]
  float* mtab;             // [N][n] emission reference of every step (written by the reference kernel)
  float* Bfwd;             // [4 slices][128 KiB] P as resident operand tiles (forward sweep)
  float* Bbwd;             // the same for P^T (backward sweep)
  float* ck;               // per CTA [n][16][128] float4: forward vectors, this CTA's 64 states
  float* part;             // per CTA [n][2 halves][128][2] partial sums (sum c gamma, sum gamma) over
                           // 32 states each, then [128][2 halves] the last forward vector's row sums
  float* w_hat;            // [N][n]
  float* marginals;        // [N][n][S] or null
  float* log_z;            // [N] or null
  int* status;
  size_t ck_stride;        // floats per CTA in ck
  size_t part_stride;      // floats per CTA in part
  float sc2;               // log2(e) / T
  int n, N;
};

// Log-transition gradient of the dense trellis (dense_dlam_kernel.cu): rows of
// X, U, V, W written by the backward kernel, one region per backward CTA
// (`region_stride` floats apart), `spr` stages of 8 rows per region.
struct DlamParams {
  const float* X;
  const float* U;
  const float* V;
  const float* W;
  float* part;             // [grid][S][S] per-CTA partial sums
  int* status;
  long long region_stride;
  long long spr;
  long long total_stages;
};

// Dense launchers (dense_kernel.cu, dense_dlam_kernel.cu).
size_t dense_smem_bytes(bool adjoint);
cudaError_t dense_geometry(bool adjoint, int n_seq, int* grid);
int dense_max_grid(bool adjoint);
cudaError_t launch_dense_prep(const float* lam, const DenseParams& p, cudaStream_t s);
cudaError_t launch_dense(const DenseParams& p, const float* lam, bool adjoint, int grid, cudaStream_t s,
                         bool prep = true);
size_t dense_tc_smem_bytes();
int dense_tc_max_clusters();
cudaError_t launch_dense_tc_forward(const DenseTCParams& p, const float* lam, int clusters, cudaStream_t s);
size_t dlam_smem_bytes();
cudaError_t dlam_grid(long long total_stages, int* grid);
cudaError_t launch_dlam(const DlamParams& p, int grid, cudaStream_t s);
cudaError_t launch_dlam_reduce(const float* part, int nparts, const float* P, float* out, int accumulate,
                               cudaStream_t s);

}  // namespace bcjr
