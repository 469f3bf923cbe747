// bitshift_kernels.cu -- hard decode, codebook-gradient reduction, and the host-side
// geometry and launches of the bitshift-trellis kernels (sm_100a).
//
// The fused forward-backward kernel itself is fb_kernel.cuh, instantiated per k
// in fb_fwd_k*.cu / fb_adj_k*.cu.
#include <cfloat>
#include <cmath>
#include <map>
#include <mutex>
#include <tuple>

#include "bcjr_device.cuh"
#include "bcjr_internal.h"
#include "team.cuh"
#include "viterbi_kernel.cuh"

namespace bcjr {

namespace {
constexpr unsigned kFull = 0xffffffffu;
}  // namespace

// grad_codebook[s] (+)= sum over teams of the per-team partials, in team order.
__global__ void gradc_reduce_kernel(const float* __restrict__ part, int num_slots, int S,
                                    float* __restrict__ out, int accumulate) {
  const int s = blockIdx.x * blockDim.x + threadIdx.x;
  if (s >= S) return;
  float acc = 0.f;
  for (int i = 0; i < num_slots; ++i) acc += part[static_cast<size_t>(i) * S + s];
  out[s] = accumulate ? out[s] + acc : acc;
}

// w_hard[i] = codebook[states[i]]: the hard codeword of every decoded state.
__global__ void gather_codewords_kernel(const int32_t* __restrict__ states, const float* __restrict__ codebook,
                                        float* __restrict__ w_hard, size_t total) {
  const size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i < total) w_hard[i] = __ldg(codebook + __ldg(states + i));
}

// ---------------------------------------------------------------------------
// Host side: geometry and launches.
// ---------------------------------------------------------------------------
const void* fb_fwd_kernel_k1(int cluster, int nseq);
const void* fb_fwd_kernel_k2(int cluster, int nseq);
const void* fb_fwd_kernel_k3(int cluster, int nseq);
const void* fb_fwd_kernel_k4(int cluster, int nseq);
const void* fb_adj_kernel_k1(int cluster, int nseq);
const void* fb_adj_kernel_k2(int cluster, int nseq);
const void* fb_adj_kernel_k3(int cluster, int nseq);
const void* fb_adj_kernel_k4(int cluster, int nseq);

namespace {

constexpr int kFBBlockThreads = 512;   // 16 states per thread, <= 128 registers per thread
constexpr int kVitBlockThreads = 512;

const void* pick_fb(bool adjoint, int k, int cl, int nseq) {
  switch (k) {
    case 1: return adjoint ? fb_adj_kernel_k1(cl, nseq) : fb_fwd_kernel_k1(cl, nseq);
    case 2: return adjoint ? fb_adj_kernel_k2(cl, nseq) : fb_fwd_kernel_k2(cl, nseq);
    case 3: return adjoint ? fb_adj_kernel_k3(cl, nseq) : fb_fwd_kernel_k3(cl, nseq);
    case 4: return adjoint ? fb_adj_kernel_k4(cl, nseq) : fb_fwd_kernel_k4(cl, nseq);
  }
  return nullptr;
}

const void* pick_viterbi(int k, int cl) {
#define BCJR_V_CASE(KK, CC, NS) \
  if (k == KK && cl == CC) return reinterpret_cast<const void*>(&viterbi_kernel<(1 << KK), CC, NS, kVitBlockThreads>);
  BCJR_V_CASE(1, 1, 1) BCJR_V_CASE(1, 2, 2) BCJR_V_CASE(1, 4, 2) BCJR_V_CASE(1, 8, 2)
  BCJR_V_CASE(2, 1, 1) BCJR_V_CASE(2, 2, 2) BCJR_V_CASE(2, 4, 2) BCJR_V_CASE(2, 8, 2)
  BCJR_V_CASE(3, 1, 1) BCJR_V_CASE(3, 2, 2) BCJR_V_CASE(3, 4, 2) BCJR_V_CASE(3, 8, 2)
  BCJR_V_CASE(4, 1, 1) BCJR_V_CASE(4, 2, 2) BCJR_V_CASE(4, 4, 2) BCJR_V_CASE(4, 8, 2)
#undef BCJR_V_CASE
  return nullptr;
}

// Team shape for a given maximum CTA size.
void base_geometry(int L, int max_block, TeamGeometry* g) {
  const int TS = (1 << L) / kStatesPerThread;
  g->team_threads = TS;
  if (TS > max_block) {
    g->block_threads = max_block;
    g->cluster = TS / max_block;
    g->teams_per_cta = 1;
  } else if (TS >= 32) {
    g->block_threads = TS;
    g->cluster = 1;
    g->teams_per_cta = 1;
  } else {
    g->block_threads = 32;
    g->cluster = 1;
    g->teams_per_cta = 32 / TS;
  }
  g->warps_per_team = TS < 32 ? 1 : TS / 32;
  g->nseq = 1;
}

int max_optin_smem() {
  int dev = 0, v = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) return 0;
  return v;
}

// Persistent grid: as many teams as can be resident, no more than there is work for.
// One kernel function serves several team sizes, so its dynamic shared-memory
// limit is raised once to the device maximum rather than to one launch's need.
cudaError_t allow_max_smem(const void* fn) {
  return cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, max_optin_smem());
}

cudaError_t persistent_grid(const void* fn, int work_units, TeamGeometry* g) {
  if (g->smem_bytes > static_cast<size_t>(max_optin_smem())) return cudaErrorNotSupported;
  cudaError_t e = allow_max_smem(fn);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  int resident_teams = 0;
  if (g->cluster > 1) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(g->cluster * sms, 1, 1);
    cfg.blockDim = dim3(g->block_threads, 1, 1);
    cfg.dynamicSmemBytes = g->smem_bytes;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = g->cluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int clusters = 0;
    if ((e = cudaOccupancyMaxActiveClusters(&clusters, fn, &cfg)) != cudaSuccess) return e;
    resident_teams = clusters;
  } else {
    int per_sm = 0;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, g->block_threads, g->smem_bytes)) !=
        cudaSuccess)
      return e;
    resident_teams = per_sm * sms * g->teams_per_cta;
  }
  if (resident_teams < 1) return cudaErrorNotSupported;
  int slots = work_units < resident_teams ? work_units : resident_teams;
  if (slots < 1) slots = 1;
  if (g->cluster > 1) {
    g->num_slots = slots;
    g->grid_blocks = slots * g->cluster;
  } else {
    const int blocks = (slots + g->teams_per_cta - 1) / g->teams_per_cta;
    g->grid_blocks = blocks;
    g->num_slots = blocks * g->teams_per_cta;
  }
  return cudaSuccess;
}

cudaError_t launch(const void* fn, const TeamGeometry& g, void** args, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(g.grid_blocks, 1, 1);
  cfg.blockDim = dim3(g.block_threads, 1, 1);
  cfg.dynamicSmemBytes = g.smem_bytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = g.cluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = g.cluster > 1 ? 1 : 0;
  return cudaLaunchKernelExC(&cfg, fn, args);
}

int states_per_thread_values(int k) {  // floats per thread in a thread-private row
  const int K = 1 << k;
  const int JT = K < 4 ? K : 4;
  const int U = K <= 4 ? 16 / (K * K) : 1;
  return U * JT;
}

}  // namespace

namespace {

// Geometry depends only on (device, sizes); computing it queries occupancy,
// so it is cached per process.
using GeoKey = std::tuple<int, int, int, int, int, int, int>;
std::mutex g_geo_mu;
std::map<GeoKey, std::pair<cudaError_t, TeamGeometry>> g_geo_cache;

cudaError_t fb_geometry_uncached(int L, int k, int n_seq, bool adjoint, int C, int nseq_request, TeamGeometry* g) {
  base_geometry(L, kFBBlockThreads, g);
  const int GL = ((1 << L) >> k) / g->cluster;
  const int NV = states_per_thread_values(k);
  const bool alias = (C == 1);
  const int max_smem = max_optin_smem();
  // Clusters keep several sequences in flight, so that the exchange wait and
  // the barrier of one sequence's step hide behind the others' steps: two by
  // default (measured fastest for both calls), or 3 or 4 on request for the
  // soft-codeword call when they fit in shared memory; k = 1 has twice the
  // group values and keeps one.
  int nseq = (g->cluster > 1 && k >= 2) ? 2 : 1;
  if (nseq_request != 0 && nseq == 2) {  // single-CTA and k = 1 teams ignore the request
    if (nseq_request < 2 || nseq_request > 4 || (adjoint && nseq_request != 2))
      return cudaErrorNotSupported;
    nseq = nseq_request;
  }
  const bool xstage = fb_xstage(g->cluster, k, nseq, adjoint, alias);
  const size_t smem =
      fb_smem_layout(GL, g->block_threads, NV, nseq, adjoint, alias, g->teams_per_cta, xstage).total;
  if (smem > static_cast<size_t>(max_smem)) return cudaErrorNotSupported;
  g->nseq = nseq;
  g->smem_bytes = smem;
  const void* fn = pick_fb(adjoint, k, g->cluster, nseq);
  if (!fn) return cudaErrorNotSupported;
  return persistent_grid(fn, (n_seq + nseq - 1) / nseq, g);
}

}  // namespace

cudaError_t fb_geometry(int L, int k, int n_seq, bool adjoint, int C, int nseq_request, TeamGeometry* g) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const GeoKey key{dev, L, k, n_seq, adjoint ? 1 : 0, C == 1 ? 1 : 0, nseq_request};
  {
    std::lock_guard<std::mutex> lk(g_geo_mu);
    auto it = g_geo_cache.find(key);
    if (it != g_geo_cache.end()) {
      *g = it->second.second;
      return it->second.first;
    }
  }
  TeamGeometry gg = {};
  e = fb_geometry_uncached(L, k, n_seq, adjoint, C, nseq_request, &gg);
  if (e == cudaSuccess || e == cudaErrorNotSupported) {
    std::lock_guard<std::mutex> lk(g_geo_mu);
    g_geo_cache[key] = {e, gg};
  }
  *g = gg;
  return e;
}

cudaError_t viterbi_geometry(int L, int k, int n_seq, TeamGeometry* g) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const GeoKey key{dev, L, k, n_seq, 2, 0, 1};
  {
    std::lock_guard<std::mutex> lk(g_geo_mu);
    auto it = g_geo_cache.find(key);
    if (it != g_geo_cache.end()) {
      *g = it->second.second;
      return it->second.first;
    }
  }
  TeamGeometry gg = {};
  base_geometry(L, kVitBlockThreads, &gg);
  const int GL = ((1 << L) >> k) / gg.cluster;
  gg.nseq = gg.cluster > 1 ? 2 : 1;  // the same as the kernel instantiations
  gg.smem_bytes = (static_cast<size_t>(gg.nseq) * (2 * GL + 2) + 192) * sizeof(double) * gg.teams_per_cta;
  if (gg.smem_bytes > static_cast<size_t>(max_optin_smem())) e = cudaErrorNotSupported;
  const void* fn = pick_viterbi(k, gg.cluster);
  if (e == cudaSuccess) e = fn ? persistent_grid(fn, (n_seq + gg.nseq - 1) / gg.nseq, &gg) : cudaErrorNotSupported;
  if (e == cudaSuccess || e == cudaErrorNotSupported) {
    std::lock_guard<std::mutex> lk(g_geo_mu);
    g_geo_cache[key] = {e, gg};
  }
  *g = gg;
  return e;
}

cudaError_t launch_fb(const FBParams& p, const TeamGeometry& g, bool adjoint, cudaStream_t s) {
  const void* fn = pick_fb(adjoint, p.k, g.cluster, g.nseq);
  if (!fn) return cudaErrorNotSupported;
  FBParams copy = p;
  void* args[] = {&copy};
  return launch(fn, g, args, s);
}

cudaError_t launch_viterbi(const ViterbiParams& p, const TeamGeometry& g, cudaStream_t s) {
  const void* fn = pick_viterbi(p.k, g.cluster);
  if (!fn) return cudaErrorNotSupported;
  ViterbiParams copy = p;
  void* args[] = {&copy};
  cudaError_t e = launch(fn, g, args, s);
  if (e != cudaSuccess || !p.w_hard) return e;
  // The hard codewords are gathered after the decode: inside it, the walker's
  // codebook load would hold up its whole warp, and with it the cluster's step.
  const size_t total = static_cast<size_t>(p.N) * p.n;
  if (total == 0) return cudaSuccess;
  const int threads = 256;
  const unsigned blocks = static_cast<unsigned>((total + threads - 1) / threads);
  gather_codewords_kernel<<<blocks, threads, 0, s>>>(p.states, p.codebook, p.w_hard, total);
  return cudaGetLastError();
}

cudaError_t launch_gradc_reduce(const float* gc_part, int num_slots, int S, float* grad_c, int accumulate,
                                cudaStream_t s) {
  const int threads = 256;
  gradc_reduce_kernel<<<(S + threads - 1) / threads, threads, 0, s>>>(gc_part, num_slots, S, grad_c,
                                                                        accumulate);
  return cudaGetLastError();
}

}  // namespace bcjr
