// bcjr_common.h -- pieces shared by the bitshift and the dense kernels.
#pragma once
#include <cuda_runtime.h>

namespace bcjr {

// Device-side error bits, OR-ed into the status word at the head of the workspace.
enum : int {
  kDevNonFinite = 1,   // log Z (or a Viterbi metric) came out NaN or infinite
  kDevTimeout = 2,     // a bounded wait gave up (the results of the call are not valid)
};

// Sum of per-team (or per-CTA) codebook-gradient partials [num_slots][S] in a
// fixed order into grad_c (added to it when `accumulate`; bitshift_kernels.cu).
cudaError_t launch_gradc_reduce(const float* gc_part, int num_slots, int S, float* grad_c,
                                int accumulate, cudaStream_t s);

}  // namespace bcjr
