// bcjr_api.cu -- the extern "C" boundary of libbcjr (declared in include/bcjr.h).
//
// Host-side only: argument validation, workspace carving, launches.  Every
// step of the computation runs in the kernels of bitshift_kernels.cu and
// dense_kernels.cu; nothing here computes on the CPU.
#include <cmath>
#include <cstring>

#include "bcjr.h"
#include "bcjr_internal.h"

using bcjr::FBParams;
using bcjr::TeamGeometry;
using bcjr::ViterbiParams;

namespace {

constexpr size_t kAlign = 256;
constexpr size_t kHeaderBytes = 256;  // int status word + padding

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Valid arguments that the bitshift kernels can run.
bcjr_status check_trellis(int L, int k) {
  if (L < 1 || k < 1 || k > L || L > 30) return BCJR_ERR_INVALID_ARG;
  if (k > 4 || 2 * k > L || L > 16 || L < 4) return BCJR_ERR_UNSUPPORTED;
  return BCJR_OK;
}

int seqs_in_flight(const bcjr_options* opt) { return opt ? opt->sequences_in_flight : 0; }

int effective_c(const bcjr_options* opt, int n) {
  int c = (opt && opt->checkpoint_interval > 0) ? opt->checkpoint_interval : 1;
  if (c > n) c = n;
  if (c < 1) c = 1;
  return c;
}

// Byte offsets of every workspace region for one bitshift call.  "Lanes" are
// the sequences in flight: teams x sequences per team.
struct FBLayout {
  size_t ck, ckR, ckF, ck64, ckF64, part, gc, total;
  size_t ck_stride, ckR_stride, ck64_stride, part_stride, row;
};

// Elements of one thread-private checkpoint row: (S/16 threads) x (forward
// values per thread); k >= 3 lanes that share a forward group keep copies.
size_t ckpt_row(int L, int k) {
  const int K = 1 << k;
  const int JT = K < 4 ? K : 4;
  const int U = K <= 4 ? 16 / (K * K) : 1;
  return (static_cast<size_t>(1) << L) / 16 * static_cast<size_t>(U * JT);
}

FBLayout fb_layout(const TeamGeometry& g, int L, int k, int n, int C, bool adjoint) {
  FBLayout l = {};
  const size_t row = ckpt_row(L, k);
  const size_t team_threads = (static_cast<size_t>(1) << L) / 16;
  const size_t lanes = static_cast<size_t>(g.num_slots) * g.nseq;
  const size_t rows = C == 1 ? static_cast<size_t>(n) : static_cast<size_t>(C);
  l.row = row;
  l.ck_stride = rows * row;
  l.ckR_stride = rows * team_threads;
  l.ck64_stride = C == 1 ? 0 : static_cast<size_t>((n - 1) / C + 1) * row;
  l.part_stride = static_cast<size_t>(n) * 2 * g.warps_per_team;
  size_t off = kHeaderBytes;
  l.ck = off;
  off = align_up(off + lanes * l.ck_stride * sizeof(float));
  l.ckR = off;
  off = align_up(off + lanes * l.ckR_stride * sizeof(uint32_t));
  l.ckF = off;
  if (adjoint) off = align_up(off + lanes * l.ck_stride * sizeof(float));
  l.ck64 = off;
  off = align_up(off + lanes * l.ck64_stride * sizeof(double));
  l.ckF64 = off;
  if (adjoint) off = align_up(off + lanes * l.ck64_stride * sizeof(float));
  l.part = off;
  off = align_up(off + lanes * l.part_stride * sizeof(float));
  l.gc = off;
  if (adjoint) off = align_up(off + static_cast<size_t>(g.num_slots) * (static_cast<size_t>(1) << L) * sizeof(float));
  l.total = off;
  return l;
}

struct ViterbiLayout {
  size_t bp, total, bp_stride;
};

ViterbiLayout viterbi_layout(const TeamGeometry& g, int L, int k, int n) {
  ViterbiLayout l = {};
  const size_t G = static_cast<size_t>(1) << (L - k);
  const int kb = k <= 2 ? k : 4;  // bits per packed backpointer (as in the kernel)
  l.bp_stride = static_cast<size_t>(n) * G * kb / 8;
  l.bp = kHeaderBytes;
  l.total = align_up(l.bp + static_cast<size_t>(g.num_slots) * g.nseq * 2 * l.bp_stride);  // two buffers per lane
  return l;
}

bcjr_status from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return BCJR_OK;
  if (e == cudaErrorNotSupported) return BCJR_ERR_UNSUPPORTED;  // needs more shared memory than a CTA has
  return BCJR_ERR_CUDA;
}

bcjr_status reset_status(void* ws, cudaStream_t s) {
  return from_cuda(cudaMemsetAsync(ws, 0, sizeof(int), s));
}

}  // namespace

// Dense entry points live in dense_api.cu.
size_t bcjr_dense_workspace_size_impl(int op, int n_states, int seq_len, int n_seq, const bcjr_options* opt);

extern "C" {

int bcjr_version(void) { return 100; }

const char* bcjr_status_string(bcjr_status s) {
  switch (s) {
    case BCJR_OK: return "BCJR_OK";
    case BCJR_ERR_INVALID_ARG: return "BCJR_ERR_INVALID_ARG: invalid argument";
    case BCJR_ERR_UNSUPPORTED: return "BCJR_ERR_UNSUPPORTED: valid but unsupported sizes";
    case BCJR_ERR_WORKSPACE: return "BCJR_ERR_WORKSPACE: workspace too small or misaligned";
    case BCJR_ERR_CUDA: return "BCJR_ERR_CUDA: CUDA runtime error";
    case BCJR_ERR_TIMEOUT: return "BCJR_ERR_TIMEOUT: a device-side wait gave up";
    case BCJR_ERR_NONFINITE: return "BCJR_ERR_NONFINITE: non-finite log-partition function or metric";
  }
  return "unknown bcjr_status";
}

size_t bcjr_workspace_size(int op, int state_bits, int k, int seq_len, int n_seq, const bcjr_options* opt) {
  if (seq_len < 1 || n_seq < 0) return 0;
  if (op == BCJR_OP_DENSE_FORWARD || op == BCJR_OP_DENSE_BACKWARD || op == BCJR_OP_DENSE_BACKWARD_LAMBDA) {
    if (state_bits < 1 || state_bits > 16) return 0;
    return bcjr_dense_workspace_size_impl(op, 1 << state_bits, seq_len, n_seq, opt);
  }
  if (check_trellis(state_bits, k) != BCJR_OK) return 0;
  const int nq = n_seq > 0 ? n_seq : 1;
  TeamGeometry g;
  if (op == BCJR_OP_FORWARD || op == BCJR_OP_BACKWARD) {
    const bool adj = op == BCJR_OP_BACKWARD;
    const int C = effective_c(opt, seq_len);
    if (bcjr::fb_geometry(state_bits, k, nq, adj, C, seqs_in_flight(opt), &g) != cudaSuccess) return 0;
    return fb_layout(g, state_bits, k, seq_len, C, adj).total;
  }
  if (op == BCJR_OP_VITERBI) {
    if (bcjr::viterbi_geometry(state_bits, k, nq, &g) != cudaSuccess) return 0;
    return viterbi_layout(g, state_bits, k, seq_len).total;
  }
  return 0;
}

static bcjr_status fb_common(bool adjoint, const float* grad_w_hat, const float* w, const float* codebook,
                             const float* w_hat_in, float T, int L, int k, int n, int N, float* w_hat,
                             float* marginals, float* log_z, float* grad_w, float* grad_c, int accumulate,
                             const bcjr_options* opt, void* ws, size_t ws_bytes, bcjr_stream_t stream) {
  bcjr_status st = check_trellis(L, k);
  if (st != BCJR_OK) return st;
  if (n < 1 || N < 0 || !(T > 0.f) || !std::isfinite(T)) return BCJR_ERR_INVALID_ARG;
  if (opt && (opt->checkpoint_interval < 0 || opt->sequences_in_flight < 0 || opt->sequences_in_flight > 4 ||
              opt->timeout_probe_cycles < 0))
    return BCJR_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int S = 1 << L;
  if (N == 0) {  // no sequences: the per-sequence arrays may be empty (null)
    if (!adjoint || accumulate) return BCJR_OK;
    if (!grad_c) return BCJR_ERR_INVALID_ARG;
    return from_cuda(cudaMemsetAsync(grad_c, 0, S * sizeof(float), s));
  }
  if (!w || !codebook || !aligned(w, 4) || !aligned(codebook, 4)) return BCJR_ERR_INVALID_ARG;
  if (adjoint) {
    if (!grad_w_hat || !w_hat_in || !grad_w || !grad_c) return BCJR_ERR_INVALID_ARG;
  } else {
    if (!w_hat) return BCJR_ERR_INVALID_ARG;
  }
  if (!ws || !aligned(ws, kAlign)) return BCJR_ERR_WORKSPACE;
  TeamGeometry g;
  const int C = effective_c(opt, n);
  if ((st = from_cuda(bcjr::fb_geometry(L, k, N, adjoint, C, seqs_in_flight(opt), &g))) != BCJR_OK) return st;
  const FBLayout lay = fb_layout(g, L, k, n, C, adjoint);
  if (ws_bytes < lay.total) return BCJR_ERR_WORKSPACE;
  char* base = static_cast<char*>(ws);
  FBParams p = {};
  p.w = w;
  p.codebook = codebook;
  p.g = grad_w_hat;
  p.what_in = w_hat_in;
  p.w_hat = w_hat;
  p.marginals = marginals;
  p.log_z = log_z;
  p.grad_w = grad_w;
  p.gc_part = reinterpret_cast<float*>(base + lay.gc);
  p.ck = reinterpret_cast<float*>(base + lay.ck);
  p.ckR = reinterpret_cast<uint32_t*>(base + lay.ckR);
  p.ckF = reinterpret_cast<float*>(base + lay.ckF);
  p.ck64 = reinterpret_cast<double*>(base + lay.ck64);
  p.ckF64 = reinterpret_cast<float*>(base + lay.ckF64);
  p.part = reinterpret_cast<float*>(base + lay.part);
  p.status = reinterpret_cast<int*>(base);
  p.ck_stride = lay.ck_stride;
  p.ckR_stride = lay.ckR_stride;
  p.ck64_stride = lay.ck64_stride;
  p.part_stride = lay.part_stride;
  p.row = lay.row;
  // the kernels carry every float64 log2-domain value times 2^128, the scaled weights and codewords times 2^64
  p.sqsc = std::ldexp(std::sqrt(1.4426950408889634 / static_cast<double>(T)), 64);
  p.two_over_T = static_cast<float>(2.0 / static_cast<double>(T));
  p.L = L;
  p.k = k;
  p.n = n;
  p.N = N;
  p.C = C;
  p.num_slots = g.num_slots;
  p.probe_wait_cycles = opt ? opt->timeout_probe_cycles : 0;
  if ((st = reset_status(ws, s)) != BCJR_OK) return st;
  if ((st = from_cuda(bcjr::launch_fb(p, g, adjoint, s))) != BCJR_OK) return st;
  if (p.probe_wait_cycles > 0 && g.cluster > 1) return BCJR_OK;  // the probe computed nothing
  if (adjoint) return from_cuda(bcjr::launch_gradc_reduce(p.gc_part, g.num_slots, S, grad_c, accumulate, s));
  return BCJR_OK;
}

bcjr_status bcjr_forward(const float* w, const float* codebook, float T, int state_bits, int k, int seq_len,
                         int n_seq, float* w_hat, float* marginals, float* log_z, const bcjr_options* opt,
                         void* workspace, size_t workspace_bytes, bcjr_stream_t stream) {
  return fb_common(false, nullptr, w, codebook, nullptr, T, state_bits, k, seq_len, n_seq, w_hat, marginals,
                   log_z, nullptr, nullptr, 0, opt, workspace, workspace_bytes, stream);
}

bcjr_status bcjr_backward(const float* grad_w_hat, const float* w, const float* codebook, const float* w_hat,
                          float T, int state_bits, int k, int seq_len, int n_seq, float* grad_w,
                          float* grad_codebook, int accumulate_codebook, const bcjr_options* opt,
                          void* workspace, size_t workspace_bytes, bcjr_stream_t stream) {
  return fb_common(true, grad_w_hat, w, codebook, w_hat, T, state_bits, k, seq_len, n_seq, nullptr, nullptr,
                   nullptr, grad_w, grad_codebook, accumulate_codebook, opt, workspace, workspace_bytes,
                   stream);
}

bcjr_status viterbi_decode(const float* w, const float* codebook, int state_bits, int k, int seq_len,
                           int n_seq, int32_t* states, float* w_hard, void* workspace, size_t workspace_bytes,
                           bcjr_stream_t stream) {
  bcjr_status st = check_trellis(state_bits, k);
  if (st != BCJR_OK) return st;
  if (seq_len < 1 || n_seq < 0) return BCJR_ERR_INVALID_ARG;
  if (n_seq == 0) return BCJR_OK;
  if (!w || !codebook || !states) return BCJR_ERR_INVALID_ARG;
  if (!workspace || !aligned(workspace, kAlign)) return BCJR_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  TeamGeometry g;
  if ((st = from_cuda(bcjr::viterbi_geometry(state_bits, k, n_seq, &g))) != BCJR_OK) return st;
  const ViterbiLayout lay = viterbi_layout(g, state_bits, k, seq_len);
  if (workspace_bytes < lay.total) return BCJR_ERR_WORKSPACE;
  char* base = static_cast<char*>(workspace);
  ViterbiParams p = {};
  p.w = w;
  p.codebook = codebook;
  p.states = states;
  p.w_hard = w_hard;
  p.metric = nullptr;
  p.bp = reinterpret_cast<uint8_t*>(base + lay.bp);
  p.status = reinterpret_cast<int*>(base);
  p.bp_stride = lay.bp_stride;
  p.L = state_bits;
  p.k = k;
  p.n = seq_len;
  p.N = n_seq;
  p.num_slots = g.num_slots;
  if ((st = reset_status(workspace, s)) != BCJR_OK) return st;
  return from_cuda(bcjr::launch_viterbi(p, g, s));
}

bcjr_status bcjr_get_status(const void* workspace, bcjr_stream_t stream) {
  if (!workspace) return BCJR_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int h = 0;
  if (cudaMemcpyAsync(&h, workspace, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess) return BCJR_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return BCJR_ERR_CUDA;
  if (h & bcjr::kDevTimeout) return BCJR_ERR_TIMEOUT;
  if (h & bcjr::kDevNonFinite) return BCJR_ERR_NONFINITE;
  return BCJR_OK;
}

}  // extern "C"
