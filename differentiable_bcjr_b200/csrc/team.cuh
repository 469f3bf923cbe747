// team.cuh -- geometry of the thread team that processes one weight sequence.
#pragma once
#include "bcjr_device.cuh"

namespace bcjr {

// Per-thread view of the team (see bcjr_device.cuh for the unit tiling).
template <int K, int CL>
struct Team {
  using TL = Tile<K>;
  int L, k, S, G, Q, TS, GL, Qc;
  int lgQc, lgGL;  // log2 of Qc and GL (all sizes are powers of two)
  int tt, lane, width, wpt, warp_in_team;
  uint32_t rank;
  int q0, j0, b0, qloc0;
  bool a_writer, b_writer;

  __device__ __forceinline__ void init(int L_, int k_, int team_thread_offset) {
    L = L_;
    k = k_;
    S = 1 << L;
    G = S >> k;
    Q = S >> (2 * k);
    TS = S / kStatesPerThread;
    GL = G / CL;
    Qc = Q / CL;
    lgQc = __ffs(Qc) - 1;
    lgGL = __ffs(GL) - 1;
    lane = threadIdx.x & 31;
    if constexpr (CL > 1) {
      rank = cluster_rank();
      tt = static_cast<int>(rank) * blockDim.x + threadIdx.x;
    } else {
      rank = 0;
      tt = threadIdx.x - team_thread_offset;
    }
    width = TS < 32 ? TS : 32;
    wpt = TS < 32 ? 1 : TS / 32;
    warp_in_team = TS < 32 ? 0 : (tt >> 5);
    if constexpr (K <= 4) {
      q0 = tt * TL::U;
      j0 = 0;
      b0 = 0;
    } else {
      q0 = tt / TL::TPU;  // compile-time power of two
      const int tile = tt % TL::TPU;
      j0 = 4 * (tile / TL::NBT);
      b0 = 4 * (tile % TL::NBT);
    }
    qloc0 = q0 - static_cast<int>(rank) * Qc;
    a_writer = (j0 == 0);
    b_writer = (b0 == 0);
  }
  __device__ __forceinline__ int state(int u, int jj, int bb) const {
    return ((j0 + jj) << (L - k)) | ((q0 + u) << k) | (b0 + bb);
  }
  // Forward-sweep exchange layout: value index i lives with the unit that reads it.
  __device__ __forceinline__ int a_read_off(int u, int jj) const { return ((j0 + jj) << lgQc) + qloc0 + u; }
  __device__ __forceinline__ void a_dest(int g, uint32_t& r, int& off) const {
    const int qq = g & (Q - 1), jj = g >> (L - 2 * k);
    r = static_cast<uint32_t>(qq >> lgQc);
    off = (jj << lgQc) | (qq & (Qc - 1));
  }
  // Backward-sweep exchange layout: contiguous blocks of G/CL values per CTA.
  __device__ __forceinline__ int b_read_off(int u, int bb) const { return (qloc0 + u) * K + b0 + bb; }
  __device__ __forceinline__ void b_dest(int h, uint32_t& r, int& off) const {
    r = static_cast<uint32_t>(h >> lgGL);
    off = h & (GL - 1);
  }
  // Output group of a forward step, and of a backward step.
  __device__ __forceinline__ int a_out_index(int u, int bb) const { return ((q0 + u) << k) | (b0 + bb); }
  __device__ __forceinline__ int b_out_index(int u, int jj) const {
    return ((j0 + jj) << (L - 2 * k)) | (q0 + u);
  }
};

}  // namespace bcjr
