// fb_fwd_k2.cu -- instantiations of the fused forward-backward kernel, k = 2 (soft codeword).
#include "fb_kernel.cuh"

namespace bcjr {

const void* fb_fwd_kernel_k2(int cluster, int nseq) {
  if (cluster == 1 && nseq == 1) return reinterpret_cast<const void*>(&fb_kernel<4, 1, false, 1, 512>);
  if (cluster == 2 && nseq == 2) return reinterpret_cast<const void*>(&fb_kernel<4, 2, false, 2, 512>);
  if (cluster == 2 && nseq == 3) return reinterpret_cast<const void*>(&fb_kernel<4, 2, false, 3, 512>);
  if (cluster == 2 && nseq == 4) return reinterpret_cast<const void*>(&fb_kernel<4, 2, false, 4, 512>);
  if (cluster == 4 && nseq == 2) return reinterpret_cast<const void*>(&fb_kernel<4, 4, false, 2, 512>);
  if (cluster == 4 && nseq == 3) return reinterpret_cast<const void*>(&fb_kernel<4, 4, false, 3, 512>);
  if (cluster == 4 && nseq == 4) return reinterpret_cast<const void*>(&fb_kernel<4, 4, false, 4, 512>);
  if (cluster == 8 && nseq == 2) return reinterpret_cast<const void*>(&fb_kernel<4, 8, false, 2, 512>);
  if (cluster == 8 && nseq == 3) return reinterpret_cast<const void*>(&fb_kernel<4, 8, false, 3, 512>);
  if (cluster == 8 && nseq == 4) return reinterpret_cast<const void*>(&fb_kernel<4, 8, false, 4, 512>);
  return nullptr;
}

}  // namespace bcjr
