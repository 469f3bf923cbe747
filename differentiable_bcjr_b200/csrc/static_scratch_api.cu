// static_scratch_api.cu -- bcjr_forward_static_scratch: the soft codeword with
// its scratch taken from a fixed, statically allocated device array instead of
// a caller-provided workspace, so that the call allocates no device memory.
//
// Why a caller may be unable to allocate: cudaMalloc and cudaFree synchronise
// the device and can take milliseconds, which a latency-bound loop that must
// keep the GPU busy cannot afford; a caller running inside an allocator's
// out-of-memory handler or a memory-pressure callback has no memory left to
// ask for; and a framework whose caching allocator owns the device's memory
// pool would fragment or oversubscribe it if a library grabbed memory beside
// it.  Such callers can still run small problems through this entry point:
// every byte it needs lives in `g_static_scratch`, which the CUDA runtime
// places in the module's global segment when the module is loaded on a device.
#include <cuda_runtime.h>

#include <mutex>

#include "bcjr.h"

namespace {

// File-scope scratch, one copy per device the module is loaded on.  Its size
// is the limit on bcjr_workspace_size(BCJR_OP_FORWARD, ...) for this entry point.
static __device__ __align__(256) unsigned char g_static_scratch[BCJR_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Address of this device's copy of the scratch, looked up once per device with
// that device current.  The first lookup may load the module on the device.
// The cached address belongs to the device's primary context: after
// cudaDeviceReset the module is loaded anew and the address may change, so a
// process that resets a device must not call these entry points on it again.
bcjr_status scratch_for_current_device(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return BCJR_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return BCJR_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_static_scratch) != cudaSuccess || !ptr) return BCJR_ERR_CUDA;
    g_scratch_ptr[dev] = ptr;
  }
  *out = g_scratch_ptr[dev];
  return BCJR_OK;
}

}  // namespace

extern "C" bcjr_status bcjr_forward_static_scratch(const float* w, const float* codebook, float T,
                                                   int state_bits, int k, int seq_len, int n_seq,
                                                   float* w_hat, float* marginals, float* log_z,
                                                   const bcjr_options* opt, bcjr_stream_t stream) {
  void* scratch = nullptr;
  const bcjr_status st = scratch_for_current_device(&scratch);
  if (st != BCJR_OK) return st;
  // The workspace path checks the size (BCJR_ERR_WORKSPACE when the problem
  // needs more than the static array holds) before it launches anything, and
  // zeroes the one word that must start at zero, the device-side status, with
  // an asynchronous memset on `stream`.  Nothing else in the scratch is read
  // before it is written.
  return bcjr_forward(w, codebook, T, state_bits, k, seq_len, n_seq, w_hat, marginals, log_z, opt, scratch,
                      BCJR_STATIC_SCRATCH_BYTES, stream);
}

extern "C" bcjr_status bcjr_static_scratch_status(bcjr_stream_t stream) {
  void* scratch = nullptr;
  const bcjr_status st = scratch_for_current_device(&scratch);
  if (st != BCJR_OK) return st;
  // The status word heads the scratch exactly as it heads a caller's workspace.
  return bcjr_get_status(scratch, stream);
}
