// fb_adj_k4.cu -- instantiations of the fused forward-backward kernel, k = 4 (vector-Jacobian product).
#include "fb_kernel.cuh"

namespace bcjr {

const void* fb_adj_kernel_k4(int cluster, int nseq) {
  if (cluster == 1 && nseq == 1) return reinterpret_cast<const void*>(&fb_kernel<16, 1, true, 1, 512>);
  if (cluster == 2 && nseq == 2) return reinterpret_cast<const void*>(&fb_kernel<16, 2, true, 2, 512>);
  if (cluster == 4 && nseq == 2) return reinterpret_cast<const void*>(&fb_kernel<16, 4, true, 2, 512>);
  if (cluster == 8 && nseq == 2) return reinterpret_cast<const void*>(&fb_kernel<16, 8, true, 2, 512>);
  return nullptr;
}

}  // namespace bcjr
