// bcjr_internal.h -- launch parameters shared by the C-ABI layer and the kernels.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace bcjr {

// Device-side error bits, OR-ed into the status word at the head of the workspace.
enum : int {
  kDevNonFinite = 1,   // log Z (or a Viterbi metric) came out NaN or infinite
  kDevTimeout = 2,     // a bounded wait gave up
};

// Geometry of one launch over the bitshift trellis (host-computed).
struct TeamGeometry {
  int team_threads;    // S / 16
  int cluster;         // CTAs per team (1 when a team fits one CTA)
  int block_threads;   // threads per CTA
  int teams_per_cta;   // > 1 only when a team is narrower than a warp
  int warps_per_team;  // max(1, team_threads / 32)
  int num_slots;       // teams resident in the grid (persistent)
  int grid_blocks;
  size_t smem_bytes;   // dynamic shared memory per CTA
};

struct FBParams {
  const float* w;          // [N][n]
  const float* codebook;   // [S]
  const float* g;          // [N][n] upstream gradient (backward)
  const float* what_in;    // [N][n] soft codeword of the forward call (backward; centring only)
  float* w_hat;            // [N][n] (forward)
  float* marginals;        // [N][n][S] or null (forward)
  float* log_z;            // [N] or null (forward)
  float* grad_w;           // [N][n] (backward)
  float* gc_part;          // [slots][S] per-team codebook-gradient partials (backward)
  float* ckpt;             // per slot [n_ckpt][G]: raw forward group vectors every C steps
  float* ckptF;            // per slot [n_ckpt][G]: forward adjoint accumulators (backward)
  float* ring;             // per slot [C][G]: recomputed segment (C > 1)
  float* ringF;            // per slot [C][G]
  float* Mst;              // per slot [n + 1]: per-step maxima used to rescale
  double* Cst;             // per slot [n + 1]: accumulated forward log2 scale
  float* part;             // per slot [n][2][warps_per_team]: per-warp partial sums
  int* status;
  size_t ckpt_stride;      // floats per slot in ckpt / ckptF
  size_t ring_stride;      // floats per slot in ring / ringF
  size_t part_stride;      // floats per slot in part
  size_t mc_stride;        // entries per slot in Mst / Cst
  float sc;                // log2(e) / T
  float two_over_T;
  int L, k, n, N, C;
  int num_slots;
};

struct ViterbiParams {
  const float* w;
  const float* codebook;
  int32_t* states;         // [N][n]
  float* w_hard;           // [N][n] or null
  double* metric;          // [N] or null
  uint8_t* bp;             // per slot [n][G] backpointers
  int* status;
  size_t bp_stride;
  int L, k, n, N;
  int num_slots;
};

// Launchers (bitshift_kernels.cu).  Return a cudaError_t from the launch.
cudaError_t launch_fb(const FBParams& p, const TeamGeometry& g, bool adjoint, cudaStream_t s);
cudaError_t launch_viterbi(const ViterbiParams& p, const TeamGeometry& g, cudaStream_t s);
cudaError_t launch_gradc_reduce(const float* gc_part, int num_slots, int S, float* grad_c,
                                int accumulate, cudaStream_t s);
// Host-side geometry: fills everything except num_slots/grid_blocks when
// `occupancy` is false; with it, also the persistent grid for this device.
cudaError_t fb_geometry(int L, int k, int n_seq, bool adjoint, TeamGeometry* g);
cudaError_t viterbi_geometry(int L, int k, int n_seq, TeamGeometry* g);

}  // namespace bcjr
