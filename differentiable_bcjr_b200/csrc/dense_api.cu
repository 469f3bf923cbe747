// dense_api.cu -- extern "C" entry points for the dense (fully connected) trellis.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "bcjr.h"
#include "dense_internal.h"

namespace {

constexpr size_t kHeader = 256;  // int status word + padding
constexpr size_t kAlign = 256;

size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

struct DenseLayout {
  size_t P, PT, ckx, ckf, ckv, ckw, mtab, gc, dlpart, total, ck_stride, mt_stride;
};

// Workspace of the vector-Jacobian product with the log-transition gradient:
// P and P^T, per CTA the rows X, U, V, W of that gradient (X and U in the
// places of the stored forward values) and the step references, the codebook
// partials, and `dl_parts` [S][S] partial sums of the row products.
DenseLayout dense_layout(int grid, int n, int dl_parts) {
  const size_t S = bcjr::kDenseStates, M = bcjr::kDenseRows;
  DenseLayout l = {};
  l.ck_stride = static_cast<size_t>(n) * M * S;
  l.mt_stride = static_cast<size_t>(n) * M;
  const size_t ck_bytes = static_cast<size_t>(grid) * l.ck_stride * sizeof(float);
  size_t off = kHeader;
  l.P = off;
  off = align_up(off + S * S * sizeof(float));
  l.PT = off;
  off = align_up(off + S * S * sizeof(float));
  l.ckx = off;
  off = align_up(off + ck_bytes);
  l.ckf = off;
  off = align_up(off + ck_bytes);
  l.ckv = off;
  off = align_up(off + ck_bytes);
  l.ckw = off;
  off = align_up(off + ck_bytes);
  l.mtab = off;
  off = align_up(off + static_cast<size_t>(grid) * l.mt_stride * sizeof(float));
  l.gc = off;
  off = align_up(off + static_cast<size_t>(grid) * S * sizeof(float));
  l.dlpart = off;
  off = align_up(off + static_cast<size_t>(dl_parts) * S * S * sizeof(float));
  l.total = off;
  return l;
}

// Workspace of the tensor-core calls: the transfer matrix as two sets of
// resident operand slices, the emission reference of every step, and per CTA
// of the resident clusters its stored forward values and partial sums (the
// adjoint adds the F~ ratios, the forward row sums and the codebook-gradient
// partials of each cluster).
struct DenseTCLayout {
  size_t Bfwd, Bbwd, mtab, ck, ckf, cks, part, gc, total, ck_stride, cks_stride, part_stride;
};

DenseTCLayout dense_tc_layout(bool adjoint, int clusters, int n, int N) {
  const size_t S = bcjr::kDenseStates, CL = bcjr::kDenseTCCluster;
  const size_t seqs = static_cast<size_t>(bcjr::dense_tc_tile_seqs(adjoint));
  DenseTCLayout l = {};
  l.ck_stride = static_cast<size_t>(n) * seqs * (S / CL);
  l.cks_stride = adjoint ? static_cast<size_t>(n) * seqs : 0;
  l.part_stride = adjoint ? static_cast<size_t>(n + 2) * 4 * seqs : static_cast<size_t>(2 * n + 1) * seqs * 2;
  const size_t ctas = static_cast<size_t>(clusters) * CL;
  size_t off = kHeader;
  l.Bfwd = off;
  off = align_up(off + S * S * 2 * sizeof(float));
  l.Bbwd = off;
  off = align_up(off + S * S * 2 * sizeof(float));
  l.mtab = off;
  off = align_up(off + static_cast<size_t>(N) * n * sizeof(float));
  l.ck = off;
  off = align_up(off + ctas * l.ck_stride * sizeof(float));
  l.ckf = off;
  if (adjoint) off = align_up(off + ctas * l.ck_stride * sizeof(float));
  l.cks = off;
  off = align_up(off + ctas * l.cks_stride * sizeof(float));
  l.part = off;
  off = align_up(off + ctas * l.part_stride * sizeof(float));
  l.gc = off;
  if (adjoint) off = align_up(off + static_cast<size_t>(clusters) * S * sizeof(float));
  l.total = off;
  return l;
}

bcjr_status dense_tc_clusters(bool adjoint, int N, int* clusters) {
  const int cap = bcjr::dense_tc_max_clusters(adjoint);
  if (cap < 1) return BCJR_ERR_UNSUPPORTED;
  const int per = bcjr::dense_tc_tile_seqs(adjoint);
  const int tiles = (N + per - 1) / per;
  *clusters = tiles < 1 ? 1 : (tiles < cap ? tiles : cap);
  return BCJR_OK;
}

// Launch geometry of the backward call that also returns the log-transition
// gradient: the rows of that gradient live in per-CTA regions, so every CTA
// takes one block of 32 sequences per launch and longer batches run in chunks
// of 32 x (CTAs that fit) sequences.  `parts` = partial sums of the reduction
// (one per SM).
bcjr_status dlam_geometry(int N, int* grid, int* chunk, int* parts) {
  const int cap = bcjr::dense_max_grid();
  if (cap < 1) return BCJR_ERR_UNSUPPORTED;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return BCJR_ERR_CUDA;
  const int blocks = (N + bcjr::kDenseRows - 1) / bcjr::kDenseRows;
  *grid = blocks < 1 ? 1 : (blocks < cap ? blocks : cap);
  *chunk = cap * bcjr::kDenseRows;
  *parts = sms;
  return BCJR_OK;
}

bcjr_status from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return BCJR_OK;
  if (e == cudaErrorNotSupported) return BCJR_ERR_UNSUPPORTED;
  return BCJR_ERR_CUDA;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// The dense kernels keep every step's forward vector (no recompute schedule).
bcjr_status check_options(const bcjr_options* opt) {
  if (!opt) return BCJR_OK;
  if (opt->checkpoint_interval < 0 || opt->sequences_in_flight != 0)
    return BCJR_ERR_INVALID_ARG;
  if (opt->checkpoint_interval > 1) return BCJR_ERR_UNSUPPORTED;
  return BCJR_OK;
}

bcjr_status dense_common(bool adjoint, const float* g, const float* w, const float* c, const float* lam,
                         const float* what_in, float T, int S, int n, int N, float* w_hat, float* marginals,
                         float* log_z, float* grad_w, float* grad_c, float* grad_lam, int accumulate,
                         const bcjr_options* opt, void* ws, size_t ws_bytes, bcjr_stream_t stream) {
  if (S < 1 || n < 1 || N < 0 || !(T > 0.f) || !std::isfinite(T)) return BCJR_ERR_INVALID_ARG;
  bcjr_status st = check_options(opt);
  if (st != BCJR_OK) return st;
  if (S != bcjr::kDenseStates) return BCJR_ERR_UNSUPPORTED;
  if (grad_lam && !aligned(grad_lam, 4)) return BCJR_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (N == 0) {
    if (!adjoint || accumulate) return BCJR_OK;
    if (!grad_c) return BCJR_ERR_INVALID_ARG;
    if (grad_lam && (st = from_cuda(cudaMemsetAsync(grad_lam, 0, S * S * sizeof(float), s))) != BCJR_OK) return st;
    return from_cuda(cudaMemsetAsync(grad_c, 0, S * sizeof(float), s));
  }
  if (!w || !c || !lam || !aligned(w, 4) || !aligned(c, 4) || !aligned(lam, 4)) return BCJR_ERR_INVALID_ARG;
  if (adjoint) {
    if (!g || !what_in || !grad_w || !grad_c) return BCJR_ERR_INVALID_ARG;
  } else {
    if (!w_hat) return BCJR_ERR_INVALID_ARG;
    if (marginals && !aligned(marginals, 16)) return BCJR_ERR_INVALID_ARG;
  }
  if (!ws || !aligned(ws, kAlign)) return BCJR_ERR_WORKSPACE;
  if (!grad_lam) {
    // The soft codeword and the plain vector-Jacobian product: the tensor-core
    // kernels (dense_tc_kernel.cu).
    int clusters = 0;
    if ((st = dense_tc_clusters(adjoint, N, &clusters)) != BCJR_OK) return st;
    const DenseTCLayout lt = dense_tc_layout(adjoint, clusters, n, N);
    if (ws_bytes < lt.total) return BCJR_ERR_WORKSPACE;
    char* b = static_cast<char*>(ws);
    bcjr::DenseTCParams tp = {};
    tp.w = w;
    tp.codebook = c;
    tp.g = g;
    tp.what_in = what_in;
    tp.mtab = reinterpret_cast<float*>(b + lt.mtab);
    tp.Bfwd = reinterpret_cast<float*>(b + lt.Bfwd);
    tp.Bbwd = reinterpret_cast<float*>(b + lt.Bbwd);
    tp.ck = reinterpret_cast<float*>(b + lt.ck);
    tp.ckf = reinterpret_cast<float*>(b + lt.ckf);
    tp.cks = reinterpret_cast<float*>(b + lt.cks);
    tp.part = reinterpret_cast<float*>(b + lt.part);
    tp.gc_part = reinterpret_cast<float*>(b + lt.gc);
    tp.w_hat = w_hat;
    tp.marginals = marginals;
    tp.log_z = log_z;
    tp.grad_w = grad_w;
    tp.status = reinterpret_cast<int*>(b);
    tp.ck_stride = lt.ck_stride;
    tp.cks_stride = lt.cks_stride;
    tp.part_stride = lt.part_stride;
    tp.sc2 = static_cast<float>(1.4426950408889634 / static_cast<double>(T));
    tp.two_over_T = static_cast<float>(2.0 / static_cast<double>(T));
    tp.n = n;
    tp.N = N;
    if ((st = from_cuda(cudaMemsetAsync(ws, 0, sizeof(int), s))) != BCJR_OK) return st;
    if ((st = from_cuda(bcjr::launch_dense_tc(tp, lam, adjoint, clusters, s))) != BCJR_OK) return st;
    if (adjoint) return from_cuda(bcjr::launch_gradc_reduce(tp.gc_part, clusters, S, grad_c, accumulate, s));
    return BCJR_OK;
  }
  // The vector-Jacobian product with the log-transition gradient (SIMT kernel
  // writing full-width rows for the tensor-core row-product sum).
  int grid = 0, chunk = N, parts = 0;
  if ((st = dlam_geometry(N, &grid, &chunk, &parts)) != BCJR_OK) return st;
  const DenseLayout lay = dense_layout(grid, n, parts);
  if (ws_bytes < lay.total) return BCJR_ERR_WORKSPACE;
  char* base = static_cast<char*>(ws);
  bcjr::DenseParams p = {};
  p.w = w;
  p.codebook = c;
  p.g = g;
  p.what_in = what_in;
  p.w_hat = w_hat;
  p.marginals = marginals;
  p.log_z = log_z;
  p.grad_w = grad_w;
  p.gc_part = reinterpret_cast<float*>(base + lay.gc);
  p.P = reinterpret_cast<const float*>(base + lay.P);
  p.PT = reinterpret_cast<const float*>(base + lay.PT);
  p.ckx = reinterpret_cast<float*>(base + lay.ckx);
  p.ckf = reinterpret_cast<float*>(base + lay.ckf);
  p.ckv = reinterpret_cast<float*>(base + lay.ckv);
  p.ckw = reinterpret_cast<float*>(base + lay.ckw);
  p.mtab = reinterpret_cast<float*>(base + lay.mtab);
  p.status = reinterpret_cast<int*>(base);
  p.ck_stride = lay.ck_stride;
  p.mt_stride = lay.mt_stride;
  p.sc2 = static_cast<float>(1.4426950408889634 / static_cast<double>(T));
  p.two_over_T = static_cast<float>(2.0 / static_cast<double>(T));
  p.n = n;
  p.N = N;
  if ((st = from_cuda(cudaMemsetAsync(ws, 0, sizeof(int), s))) != BCJR_OK) return st;
  // Backward call with the log-transition gradient, chunk by chunk: each
  // chunk's backward kernel writes the rows X, U, V, W of its transitions, the
  // tensor-core kernel sums them into per-SM partials, and the reductions add
  // the chunk's codebook and log-transition gradients to the outputs.
  float* dlpart = reinterpret_cast<float*>(base + lay.dlpart);
  for (int c0 = 0; c0 < N; c0 += chunk) {
    const int Nc = (N - c0) < chunk ? (N - c0) : chunk;
    const int acc = (accumulate || c0 > 0) ? 1 : 0;
    const size_t off = static_cast<size_t>(c0) * n;
    bcjr::DenseParams pc = p;
    pc.w = w + off;
    pc.g = g + off;
    pc.what_in = what_in + off;
    pc.grad_w = grad_w + off;
    pc.N = Nc;
    const int grid_c = (Nc + bcjr::kDenseRows - 1) / bcjr::kDenseRows;
    if ((st = from_cuda(bcjr::launch_dense(pc, lam, grid_c, s, c0 == 0))) != BCJR_OK) return st;
    if ((st = from_cuda(bcjr::launch_gradc_reduce(pc.gc_part, grid_c, S, grad_c, acc, s))) != BCJR_OK) return st;
    if (n == 1) {  // no transitions: the gradient is zero
      if (!acc && (st = from_cuda(cudaMemsetAsync(grad_lam, 0, S * S * sizeof(float), s))) != BCJR_OK) return st;
      continue;
    }
    bcjr::DlamParams dp = {};
    dp.X = pc.ckx;
    dp.U = pc.ckf;
    dp.V = pc.ckv;
    dp.W = pc.ckw;
    dp.part = dlpart;
    dp.status = pc.status;
    dp.region_stride = static_cast<long long>(lay.ck_stride);
    dp.spr = static_cast<long long>(n - 1) * (bcjr::kDenseRows / 8);
    dp.total_stages = static_cast<long long>(grid_c) * dp.spr;
    int gd = 0;
    if ((st = from_cuda(bcjr::dlam_grid(dp.total_stages, &gd))) != BCJR_OK) return st;
    if (gd > parts) gd = parts;
    if ((st = from_cuda(bcjr::launch_dlam(dp, gd, s))) != BCJR_OK) return st;
    if ((st = from_cuda(bcjr::launch_dlam_reduce(dlpart, gd, pc.P, grad_lam, acc, s))) != BCJR_OK) return st;
  }
  return BCJR_OK;
}

}  // namespace

size_t bcjr_dense_workspace_size_impl(int op, int n_states, int seq_len, int n_seq, const bcjr_options* opt) {
  if (n_states != bcjr::kDenseStates || seq_len < 1 || n_seq < 0) return 0;
  if (check_options(opt) != BCJR_OK) return 0;
  const bool adjoint = (op == BCJR_OP_DENSE_BACKWARD || op == BCJR_OP_DENSE_BACKWARD_LAMBDA);
  int grid = 0;
  if (op == BCJR_OP_DENSE_BACKWARD_LAMBDA) {
    int chunk = 0, parts = 0;
    if (dlam_geometry(n_seq > 0 ? n_seq : 1, &grid, &chunk, &parts) != BCJR_OK) return 0;
    return dense_layout(grid, seq_len, parts).total;
  }
  int clusters = 0;
  if (dense_tc_clusters(adjoint, n_seq > 0 ? n_seq : 1, &clusters) != BCJR_OK) return 0;
  return dense_tc_layout(adjoint, clusters, seq_len, n_seq > 0 ? n_seq : 1).total;
}

extern "C" {

bcjr_status bcjr_dense_forward(const float* w, const float* codebook, const float* log_trans, float T,
                               int n_states, int seq_len, int n_seq, float* w_hat, float* marginals,
                               float* log_z, const bcjr_options* opt, void* workspace, size_t workspace_bytes,
                               bcjr_stream_t stream) {
  return dense_common(false, nullptr, w, codebook, log_trans, nullptr, T, n_states, seq_len, n_seq, w_hat,
                      marginals, log_z, nullptr, nullptr, nullptr, 0, opt, workspace, workspace_bytes, stream);
}

bcjr_status bcjr_dense_backward(const float* grad_w_hat, const float* w, const float* codebook,
                                const float* log_trans, const float* w_hat, float T, int n_states, int seq_len,
                                int n_seq, float* grad_w, float* grad_codebook, int accumulate_codebook,
                                const bcjr_options* opt, void* workspace, size_t workspace_bytes,
                                bcjr_stream_t stream) {
  return dense_common(true, grad_w_hat, w, codebook, log_trans, w_hat, T, n_states, seq_len, n_seq, nullptr,
                      nullptr, nullptr, grad_w, grad_codebook, nullptr, accumulate_codebook, opt, workspace,
                      workspace_bytes, stream);
}

bcjr_status bcjr_dense_backward_lambda(const float* grad_w_hat, const float* w, const float* codebook,
                                       const float* log_trans, const float* w_hat, float T, int n_states,
                                       int seq_len, int n_seq, float* grad_w, float* grad_codebook,
                                       float* grad_log_trans, int accumulate, const bcjr_options* opt,
                                       void* workspace, size_t workspace_bytes, bcjr_stream_t stream) {
  if (!grad_log_trans) return BCJR_ERR_INVALID_ARG;
  return dense_common(true, grad_w_hat, w, codebook, log_trans, w_hat, T, n_states, seq_len, n_seq, nullptr,
                      nullptr, nullptr, grad_w, grad_codebook, grad_log_trans, accumulate, opt, workspace,
                      workspace_bytes, stream);
}

}  // extern "C"
