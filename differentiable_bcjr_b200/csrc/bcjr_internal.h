// bcjr_internal.h -- launch parameters shared by the C-ABI layer and the kernels.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "bcjr_common.h"

namespace bcjr {



// Geometry of one launch over the bitshift trellis (host-computed).
struct TeamGeometry {
  int team_threads;    // S / 16
  int cluster;         // CTAs per team (1 when a team fits one CTA)
  int block_threads;   // threads per CTA
  int teams_per_cta;   // > 1 only when a team is narrower than a warp
  int warps_per_team;  // max(1, team_threads / 32)
  int nseq;            // sequences in flight per team (forward-backward kernels)
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
  // Per sequence in flight ("lane" = slot * nseq + x).  Rows are thread-private:
  // thread tt of the team owns elements [tt*NV, tt*NV + NV) of every row, so a
  // row holds team_threads * NV values (= S/2^k for k <= 2, S/4 for k >= 3,
  // where lanes sharing a forward group each keep their own copy).
  // Forward values A_t (every float64 log2-domain value carries a factor 2^128):
  float* ck;               // C == 1: [n][row] A_t - R (float, unscaled); C > 1: ring [C][row]
  uint32_t* ckR;           // [n][team_threads] high word of each thread's reference R - 1; C > 1: ring
  float* ckF;              // backward: same layout as ck for the forward adjoint accumulators
  double* ck64;            // C > 1: [n/C + 1][row] A'_t at t = 0, C, 2C, ... (float64)
  float* ckF64;            // C > 1: [n/C + 1][row] forward adjoint accumulators at the same t
  float* part;             // [n][2][warps_per_team] per-warp partial sums
  int* status;
  size_t ck_stride;        // floats per lane in ck / ckF
  size_t ckR_stride;       // words per lane in ckR
  size_t ck64_stride;      // elements per lane in ck64 / ckF64
  size_t part_stride;      // floats per lane in part
  size_t row;              // elements per checkpoint row (team_threads * NV)
  double sqsc;             // sqrt(log2(e) / T) * 2^64: emission phi * 2^128 = -((w - c) sqsc)^2
  float two_over_T;
  int L, k, n, N, C;
  int num_slots;
  long long probe_wait_cycles;  // > 0: only the bounded-wait probe runs (testing aid)
};

// Whether a forward-backward launch stages its outgoing forward-sweep values
// for bulk copies (fb_kernel's xst_on): cluster teams with k <= 2 and up to
// two sequences in flight; the adjoint only with C = 1 (`alias`).
__host__ __device__ inline bool fb_xstage(int cluster, int k, int nseq, bool adj, bool alias) {
  return cluster > 1 && k <= 2 && nseq <= 2 && (!adj || alias);
}

// Shared-memory carve-up of the forward-backward kernel (bytes), identical on
// host and device.  Per team and per sequence in flight: the double-buffered
// exchange vectors (float64 group values, float32 adjoint accumulators); per
// CTA: a reduction scratch, the thread-private staging of the forward
// values read by the backward sweep (values, reference words, accumulators),
// and every thread's float codewords.
struct FBSmem {
  uint32_t exA, exF, exB, exBt, mbar, per_seq, per_team, red, stage, stageK, stageF, xst, xstF, cf, total;
};
// `xstage`: outgoing group values are staged per sequence in flight and
// parity (GL float64, and GL float32 accumulators for the adjoint) and leave
// by bulk copy.  The adjoint stages its forward sweep only, so its staging
// shares room with the checkpoint staging, which only its backward sweep uses.
__host__ __device__ inline FBSmem fb_smem_layout(int GL, int NT, int NV, int nseq, bool adj, bool alias,
                                                 int teams_per_cta, bool xstage) {
  FBSmem l;
  uint32_t o = 0;
  l.exA = o;
  o += 2u * GL * 8u;
  l.exF = o;
  if (adj) o += 2u * GL * 4u;
  l.exB = alias ? l.exA : o;
  if (!alias) o += 2u * GL * 8u;
  l.exBt = alias ? l.exF : o;
  if (!alias && adj) o += 2u * GL * 4u;
  o = (o + 15u) & ~15u;
  l.mbar = o;  // 2 sets (forward / backward buffers) x 2 parities of 8-byte mbarriers
  o += 32u;
  l.per_seq = o;
  l.per_team = static_cast<uint32_t>(nseq) * o;
  l.red = static_cast<uint32_t>(teams_per_cta) * l.per_team;
  o = l.red + 4u * 128u * 4u;
  // staging of the stored forward values (C == 1 only; C > 1 reads its ring
  // directly): NV floats, one reference word and (adjoint) NV accumulators
  const uint32_t stg = alias ? static_cast<uint32_t>(nseq) * NT : 0u;  // one slot per sequence in flight
  l.stage = o;
  o += stg * NV * 4u;
  l.stageF = o;
  if (adj) o += stg * NV * 4u;
  l.stageK = o;
  o += stg * 4u;
  o = (o + 15u) & ~15u;
  l.xst = adj ? l.stage : o;
  l.xstF = l.xst + static_cast<uint32_t>(nseq) * 2u * GL * 8u;
  const uint32_t xend = l.xstF + (adj ? static_cast<uint32_t>(nseq) * 2u * GL * 4u : 0u);
  if (xstage && xend > o) o = (xend + 15u) & ~15u;
  l.cf = o;  // float codewords of every thread: [8 pairs][NT] float2
  o += static_cast<uint32_t>(NT) * 16u * 4u;
  l.total = o;
  return l;
}

struct ViterbiParams {
  const float* w;
  const float* codebook;
  int32_t* states;         // [N][n]
  float* w_hard;           // [N][n] or null
  double* metric;          // [N] or null
  uint8_t* bp;             // per lane (slot x sequence in flight) [2][n][G x kb bits] packed backpointers (by iteration parity)
  int* status;
  size_t bp_stride;
  int L, k, n, N;
  int num_slots;
};

// Launchers (bitshift_kernels.cu).  Return a cudaError_t from the launch.
cudaError_t launch_fb(const FBParams& p, const TeamGeometry& g, bool adjoint, cudaStream_t s);
cudaError_t launch_viterbi(const ViterbiParams& p, const TeamGeometry& g, cudaStream_t s);
// Host-side geometry and persistent grid for this device.  cudaErrorNotSupported
// when no configuration fits the shared memory of one CTA.
cudaError_t fb_geometry(int L, int k, int n_seq, bool adjoint, int C, int nseq_request, TeamGeometry* g);
cudaError_t viterbi_geometry(int L, int k, int n_seq, TeamGeometry* g);

}  // namespace bcjr
