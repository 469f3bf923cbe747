// fb_fwd_k1.cu -- instantiations of the fused forward-backward kernel, k = 1 (soft codeword).
#include "fb_kernel.cuh"

namespace bcjr {

const void* fb_fwd_kernel_k1(int cluster, int nseq) {
  if (cluster == 1 && nseq == 1) return reinterpret_cast<const void*>(&fb_kernel<2, 1, false, 1, 512>);
  if (cluster == 2 && nseq == 1) return reinterpret_cast<const void*>(&fb_kernel<2, 2, false, 1, 512>);
  if (cluster == 4 && nseq == 1) return reinterpret_cast<const void*>(&fb_kernel<2, 4, false, 1, 512>);
  if (cluster == 8 && nseq == 1) return reinterpret_cast<const void*>(&fb_kernel<2, 8, false, 1, 512>);
  return nullptr;
}

}  // namespace bcjr
