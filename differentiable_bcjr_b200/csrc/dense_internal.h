// dense_internal.h -- launch parameters of the dense (fully connected) trellis
// kernels, shared by the C-ABI layer and the kernels.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "bcjr_common.h"

namespace bcjr {

// Dense (fully connected) trellis: 256 states.
constexpr int kDenseStates = 256;

// The dense trellis on the tensor cores (dense_tc_kernel.cu): a cluster of
// kDenseTCCluster CTAs per tile of kDenseTCRows MMA rows, CTA r holding K-slice
// r of the transfer matrix.  The soft-codeword call puts one sequence on each
// row (128 per tile); the vector-Jacobian product stacks each sequence's two
// operands on adjacent rows (64 sequences per tile).
constexpr int kDenseTCCluster = 4;
constexpr int kDenseTCRows = 128;

struct DenseTCParams {
  const float* w;          // [N][n]
  const float* codebook;   // [S]
  const float* g;          // [N][n] upstream gradient (vector-Jacobian product)
  const float* what_in;    // [N][n] soft codeword of the forward call (vector-Jacobian product)
  float* mtab;             // [N][n] emission reference of every step (written by the reference kernel)
  float* Bfwd;             // [4 slices][128 KiB] P as resident operand tiles (forward sweep)
  float* Bbwd;             // the same for P^T (backward sweep)
  float* ck;               // per CTA: forward vectors of this CTA's 64 states, every step
  float* ckf;              // per CTA: forward adjoint ratios F~ (vector-Jacobian product)
  float* cks;              // per CTA [n][64]: every step's forward row sum (vector-Jacobian product)
  float* part;             // per CTA: per-row partial sums over its states (layouts in the kernel)
  float* w_hat;            // [N][n] (soft codeword)
  float* marginals;        // [N][n][S] or null (soft codeword)
  float* log_z;            // [N] or null (soft codeword)
  float* grad_w;           // [N][n] (vector-Jacobian product)
  float* gc_part;          // [clusters][S] codebook-gradient partials (vector-Jacobian product)
  float* P;                // [S][S] exp(Lambda) row-major, or null (written by the prep kernel)
  // Rows of the log-transition gradient (vector-Jacobian product, or null):
  // per cluster a region of [n - 1][64 sequences][S] rows, row (t, q) for the
  // transition t -> t + 1; each CTA writes its 64 states of every row.
  float* rowX;
  float* rowU;
  float* rowV;
  float* rowW;
  size_t row_region;       // floats per cluster region of each row array
  int* status;
  size_t ck_stride;        // floats per CTA in ck and ckf
  size_t cks_stride;       // floats per CTA in cks
  size_t part_stride;      // floats per CTA in part
  float sc2;               // log2(e) / T
  float two_over_T;
  int n, N;
};

// Log-transition gradient of the dense trellis (dense_dlam_kernel.cu): rows of
// X, U, V, W written by the tensor-core adjoint, one region per cluster
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

// Launchers (dense_tc_kernel.cu, dense_dlam_kernel.cu).
size_t dense_tc_smem_bytes();
int dense_tc_max_clusters(bool adjoint);
// Sequences per cluster tile: 128 for the soft codeword, 64 for the adjoint.
constexpr int dense_tc_tile_seqs(bool adjoint) { return adjoint ? kDenseTCRows / 2 : kDenseTCRows; }
cudaError_t launch_dense_tc(const DenseTCParams& p, const float* lam, bool adjoint, int clusters, cudaStream_t s);
size_t dlam_smem_bytes();
cudaError_t dlam_grid(long long total_stages, int* grid);
cudaError_t launch_dlam(const DlamParams& p, int grid, cudaStream_t s);
cudaError_t launch_dlam_reduce(const float* part, int nparts, const float* P, float* out, int accumulate,
                               cudaStream_t s);

}  // namespace bcjr
