// dense_api.cu -- dense (fully connected) trellis entry points.
#include "bcjr.h"
#include "bcjr_internal.h"

size_t bcjr_dense_workspace_size_impl(int op, int n_states, int seq_len, int n_seq, const bcjr_options* opt) {
  (void)op; (void)n_states; (void)seq_len; (void)n_seq; (void)opt;
  return 0;
}

extern "C" {

bcjr_status bcjr_dense_forward(const float*, const float*, const float*, float, int, int, int, float*, float*,
                               float*, const bcjr_options*, void*, size_t, bcjr_stream_t) {
  return BCJR_ERR_UNSUPPORTED;
}

bcjr_status bcjr_dense_backward(const float*, const float*, const float*, const float*, const float*, float, int,
                                int, int, float*, float*, int, const bcjr_options*, void*, size_t,
                                bcjr_stream_t) {
  return BCJR_ERR_UNSUPPORTED;
}

}  // extern "C"
