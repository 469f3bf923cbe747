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

namespace bcjr {

namespace {
constexpr unsigned kFull = 0xffffffffu;
}  // namespace

// ---------------------------------------------------------------------------
// Hard decode: max-sum over -(w - c)^2 in float64, each difference, square and
// sum rounded separately, ties to the lowest predecessor index and the lowest
// final state ("BCJR-QAT", technical summary: T -> 0 recovers the hard Viterbi
// output).  Backpointers (k bits, stored as bytes) go to the workspace; one
// thread of the team walks them back.
// ---------------------------------------------------------------------------
template <int K, int CL, int NTB>
__global__ void __launch_bounds__(NTB, 1) viterbi_kernel(const ViterbiParams p) {
  using TL = Tile<K>;
  constexpr int U = TL::U, JT = TL::JT, BT = TL::BT;
  const int L = p.L, k = p.k, n = p.n;
  const int S = 1 << L;
  const int TS = S / kStatesPerThread;
  const int tpc = (CL == 1 && TS < static_cast<int>(blockDim.x)) ? static_cast<int>(blockDim.x) / TS : 1;
  const int team_in_cta = (tpc > 1) ? static_cast<int>(threadIdx.x) / TS : 0;
  Team<K, CL> tm;
  tm.init(L, k, team_in_cta * TS);
  const int slot = (CL > 1) ? static_cast<int>(blockIdx.x) / CL : static_cast<int>(blockIdx.x) * tpc + team_in_cta;
  const int G = tm.G, GL = tm.GL;

  extern __shared__ __align__(16) double smemd[];
  double* base = smemd + team_in_cta * (2 * static_cast<size_t>(GL) + 2 * 128);
  double* bufV = base;                 // [2][GL]
  double* redv = bufV + 2 * GL;        // [128]
  int* reds = reinterpret_cast<int*>(redv + 128);  // [128]

  float cb[U][JT][BT];
#pragma unroll
  for (int u = 0; u < U; ++u)
#pragma unroll
    for (int jj = 0; jj < JT; ++jj)
#pragma unroll
      for (int bb = 0; bb < BT; ++bb) cb[u][jj][bb] = __ldg(p.codebook + tm.state(u, jj, bb));

  uint8_t* bp = p.bp + static_cast<size_t>(slot) * p.bp_stride;
  // Every CTA of the cluster must be running before any of them writes into
  // another's shared memory.
  if constexpr (CL > 1) cluster_sync_all();
  const int iters = (p.N + p.num_slots - 1) / p.num_slots;
  for (int it = 0; it < iters; ++it) {
    const int seq_raw = slot + it * p.num_slots;
    const bool active = seq_raw < p.N;
    const int seq = active ? seq_raw : p.N - 1;
    const float* wseq = p.w + static_cast<size_t>(seq) * n;
    double best[U][BT];
    int bj[U][BT];
    for (int t = 0; t < n; ++t) {
      const double wt = static_cast<double>(__ldg(wseq + t));
      double a[U][JT];
#pragma unroll
      for (int u = 0; u < U; ++u)
#pragma unroll
        for (int jj = 0; jj < JT; ++jj)
          a[u][jj] = (t == 0) ? 0.0 : bufV[(t & 1) * GL + tm.a_read_off(u, jj)];
#pragma unroll
      for (int u = 0; u < U; ++u)
#pragma unroll
        for (int bb = 0; bb < BT; ++bb) {
          double bv = -DBL_MAX;
          int bjj = 0;
#pragma unroll
          for (int jj = 0; jj < JT; ++jj) {
            const double d = __dsub_rn(wt, static_cast<double>(cb[u][jj][bb]));
            const double v = __dadd_rn(a[u][jj], -__dmul_rn(d, d));
            if (jj == 0 || v > bv) {
              bv = v;
              bjj = tm.j0 + jj;
            }
          }
          if constexpr (K >= 8) {
#pragma unroll
            for (int o = TL::NBT; o < TL::TPU; o <<= 1) {
              const double ov = __shfl_xor_sync(kFull, bv, o);
              const int oj = __shfl_xor_sync(kFull, bjj, o);
              if (ov > bv || (ov == bv && oj < bjj)) {
                bv = ov;
                bjj = oj;
              }
            }
          }
          best[u][bb] = bv;
          bj[u][bb] = bjj;
        }
      if (t + 1 < n && tm.a_writer) {
        uint8_t* brow = bp + static_cast<size_t>(t + 1) * G;
#pragma unroll
        for (int u = 0; u < U; ++u)
#pragma unroll
          for (int bb = 0; bb < BT; ++bb) {
            const int gi = tm.a_out_index(u, bb);
            uint32_t r;
            int off;
            tm.a_dest(gi, r, off);
            team_store_f64<CL>(bufV + ((t + 1) & 1) * GL, r, off, best[u][bb]);
            brow[gi] = static_cast<uint8_t>(bj[u][bb]);
          }
      }
      team_sync<CL>();
    }
    // End state: the largest final metric, lowest state on ties.
    double vb = -DBL_MAX;
    int sb = S;  // S marks "no candidate"; every reduction below keeps a valid state when one exists
    if (tm.a_writer) {
#pragma unroll
      for (int u = 0; u < U; ++u)
#pragma unroll
        for (int bb = 0; bb < BT; ++bb) {
          const int st = (bj[u][bb] << (L - k)) | tm.a_out_index(u, bb);
          if (sb == S || best[u][bb] > vb || (best[u][bb] == vb && st < sb)) {
            vb = best[u][bb];
            sb = st;
          }
        }
    }
    for (int o = tm.width >> 1; o > 0; o >>= 1) {
      const double ov = __shfl_xor_sync(kFull, vb, o);
      const int os = __shfl_xor_sync(kFull, sb, o);
      if (os != S && (sb == S || ov > vb || (ov == vb && os < sb))) {
        vb = ov;
        sb = os;
      }
    }
    if (tm.TS > 32) {
      if (tm.lane == 0) {
        for (int r = 0; r < CL; ++r) {
          team_store_f64<CL>(redv, r, tm.warp_in_team, vb);
          team_store_u32<CL>(reinterpret_cast<uint32_t*>(reds), r, tm.warp_in_team, static_cast<uint32_t>(sb));
        }
      }
      team_sync<CL>();
      vb = -DBL_MAX;
      sb = S;
      for (int i = 0; i < tm.wpt; ++i) {
        const double ov = redv[i];
        const int os = reds[i];
        if (os != S && (sb == S || ov > vb || (ov == vb && os < sb))) {
          vb = ov;
          sb = os;
        }
      }
    }
    // Non-finite metrics (NaN inputs) can leave no comparable candidate: keep the walk in range.
    if (sb < 0 || sb >= S) sb = 0;
    if (tm.tt == 0 && active) {
      if (!isfinite(vb)) atomicOr(p.status, kDevNonFinite);
      if (p.metric) p.metric[seq] = vb;
      int s = sb;
      int32_t* st = p.states + static_cast<size_t>(seq) * n;
      float* wh = p.w_hard ? p.w_hard + static_cast<size_t>(seq) * n : nullptr;
      for (int t = n - 1; t >= 0; --t) {
        st[t] = s;
        if (wh) wh[t] = __ldg(p.codebook + s);
        if (t >= 1) {
          const int j = bp[static_cast<size_t>(t) * G + (s >> k)];
          s = (j << (L - k)) | (s >> k);
        }
      }
    }
    team_sync<CL>();
  }
  if constexpr (CL > 1) cluster_sync_all();
}

// grad_codebook[s] (+)= sum over teams of the per-team partials, in team order.
__global__ void gradc_reduce_kernel(const float* __restrict__ part, int num_slots, int S,
                                    float* __restrict__ out, int accumulate) {
  const int s = blockIdx.x * blockDim.x + threadIdx.x;
  if (s >= S) return;
  float acc = 0.f;
  for (int i = 0; i < num_slots; ++i) acc += part[static_cast<size_t>(i) * S + s];
  out[s] = accumulate ? out[s] + acc : acc;
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

constexpr int kFBBlockThreads = 512;  // 16 states per thread, <= 128 registers per thread

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
#define BCJR_V_CASE(KK, CC) \
  if (k == KK && cl == CC) return reinterpret_cast<const void*>(&viterbi_kernel<(1 << KK), CC, 1024>);
  BCJR_V_CASE(1, 1) BCJR_V_CASE(1, 2) BCJR_V_CASE(1, 4)
  BCJR_V_CASE(2, 1) BCJR_V_CASE(2, 2) BCJR_V_CASE(2, 4)
  BCJR_V_CASE(3, 1) BCJR_V_CASE(3, 2) BCJR_V_CASE(3, 4)
  BCJR_V_CASE(4, 1) BCJR_V_CASE(4, 2) BCJR_V_CASE(4, 4)
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
  (void)nseq_request;
  // Clusters keep two sequences in flight (the barrier of one hides behind the
  // other's step); k = 1 has twice the group values and keeps one.
  const int nseq = (g->cluster > 1 && k >= 2) ? 2 : 1;
  const size_t smem = fb_smem_layout(GL, g->block_threads, NV, nseq, adjoint, alias, g->teams_per_cta).total;
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
  const GeoKey key{dev, L, k, n_seq, adjoint ? 1 : 0, C == 1 ? 1 : 0, nseq_request == 1 ? 3 : 0};
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
  base_geometry(L, 1024, &gg);
  const int GL = ((1 << L) >> k) / gg.cluster;
  gg.smem_bytes = (2 * static_cast<size_t>(GL) + 2 * 128) * sizeof(double) * gg.teams_per_cta;
  const void* fn = pick_viterbi(k, gg.cluster);
  e = fn ? persistent_grid(fn, n_seq, &gg) : cudaErrorNotSupported;
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
  return launch(fn, g, args, s);
}

cudaError_t launch_gradc_reduce(const float* gc_part, int num_slots, int S, float* grad_c, int accumulate,
                                cudaStream_t s) {
  const int threads = 256;
  gradc_reduce_kernel<<<(S + threads - 1) / threads, threads, 0, s>>>(gc_part, num_slots, S, grad_c,
                                                                        accumulate);
  return cudaGetLastError();
}

}  // namespace bcjr
