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

// Workspace of the tensor-core calls: the transfer matrix as two sets of
// resident operand slices, the emission reference of every step, and per CTA
// of the resident clusters its stored forward values and partial sums (the
// adjoint adds the F~ ratios, the forward row sums and the codebook-gradient
// partials of each cluster).  With the log-transition gradient it adds P
// row-major, the rows X, U, V, W of every cluster's tile and `dl_parts`
// [S][S] partial sums of their products.
struct DenseTCLayout {
  size_t Bfwd, Bbwd, mtab, ck, ckf, cks, part, gc, P, rows, dlpart, total;
  size_t ck_stride, cks_stride, part_stride, row_region;
};

DenseTCLayout dense_tc_layout(bool adjoint, int clusters, int n, int N, int dl_parts) {
  const size_t S = bcjr::kDenseStates, CL = bcjr::kDenseTCCluster;
  const size_t seqs = static_cast<size_t>(bcjr::dense_tc_tile_seqs(adjoint));
  DenseTCLayout l = {};
  l.ck_stride = static_cast<size_t>(n) * seqs * (S / CL);
  l.cks_stride = adjoint ? static_cast<size_t>(n) * seqs : 0;
  l.part_stride = adjoint ? static_cast<size_t>(n + 2) * 4 * seqs : static_cast<size_t>(2 * n + 1) * seqs * 2;
  l.row_region = dl_parts > 0 ? static_cast<size_t>(n - 1) * seqs * S : 0;
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
  l.P = off;
  if (dl_parts > 0) off = align_up(off + S * S * sizeof(float));
  l.rows = off;
  off = align_up(off + 4 * static_cast<size_t>(clusters) * l.row_region * sizeof(float));
  l.dlpart = off;
  off = align_up(off + static_cast<size_t>(dl_parts) * S * S * sizeof(float));
  l.total = off;
  return l;
}

// Clusters of one launch: one per tile, at most as many as fit.
bcjr_status dense_tc_clusters(bool adjoint, int N, int* clusters) {
  const int cap = bcjr::dense_tc_max_clusters(adjoint);
  if (cap < 1) return BCJR_ERR_UNSUPPORTED;
  const int per = bcjr::dense_tc_tile_seqs(adjoint);
  const int tiles = (N + per - 1) / per;
  *clusters = tiles < 1 ? 1 : (tiles < cap ? tiles : cap);
  return BCJR_OK;
}

// Partial sums of the log-transition gradient's row-product sum: one per SM.
bcjr_status dlam_parts(int* parts) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(parts, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return BCJR_ERR_CUDA;
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
  // All three calls run the tensor-core kernels (dense_tc_kernel.cu).  With
  // the log-transition gradient the adjoint runs in chunks of one tile per
  // cluster, writing the rows X, U, V, W of each chunk's transitions, which the
  // tensor-core row-product sum (dense_dlam_kernel.cu) adds up after each chunk.
  const bool dl = grad_lam != nullptr;
  int clusters = 0, parts = 0;
  if ((st = dense_tc_clusters(adjoint, N, &clusters)) != BCJR_OK) return st;
  if (dl && (st = dlam_parts(&parts)) != BCJR_OK) return st;
  const int per = bcjr::dense_tc_tile_seqs(adjoint);
  const int chunk = dl ? clusters * per : N;
  const DenseTCLayout lt = dense_tc_layout(adjoint, clusters, n, chunk < N ? chunk : N, dl ? parts : 0);
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
  if (!dl) {
    if ((st = from_cuda(bcjr::launch_dense_tc(tp, lam, adjoint, clusters, s))) != BCJR_OK) return st;
    if (adjoint) return from_cuda(bcjr::launch_gradc_reduce(tp.gc_part, clusters, S, grad_c, accumulate, s));
    return BCJR_OK;
  }
  float* rows = reinterpret_cast<float*>(b + lt.rows);
  const size_t rstride = static_cast<size_t>(clusters) * lt.row_region;
  if (n > 1) {
    tp.P = reinterpret_cast<float*>(b + lt.P);
    tp.rowX = rows;
    tp.rowU = rows + rstride;
    tp.rowV = rows + 2 * rstride;
    tp.rowW = rows + 3 * rstride;
    tp.row_region = lt.row_region;
  }
  float* dlpart = reinterpret_cast<float*>(b + lt.dlpart);
  for (int c0 = 0; c0 < N; c0 += chunk) {
    const int Nc = (N - c0) < chunk ? (N - c0) : chunk;
    const int acc = (accumulate || c0 > 0) ? 1 : 0;
    const size_t off = static_cast<size_t>(c0) * n;
    bcjr::DenseTCParams pc = tp;
    pc.w = w + off;
    pc.g = g + off;
    pc.what_in = what_in + off;
    pc.grad_w = grad_w + off;
    pc.N = Nc;
    const int cl_c = (Nc + per - 1) / per;
    if ((st = from_cuda(bcjr::launch_dense_tc(pc, lam, true, cl_c, s))) != BCJR_OK) return st;
    if ((st = from_cuda(bcjr::launch_gradc_reduce(pc.gc_part, cl_c, S, grad_c, acc, s))) != BCJR_OK) return st;
    if (n == 1) {  // no transitions: the gradient is zero
      if (!acc && (st = from_cuda(cudaMemsetAsync(grad_lam, 0, S * S * sizeof(float), s))) != BCJR_OK) return st;
      continue;
    }
    bcjr::DlamParams dp = {};
    dp.X = pc.rowX;
    dp.U = pc.rowU;
    dp.V = pc.rowV;
    dp.W = pc.rowW;
    dp.part = dlpart;
    dp.status = pc.status;
    dp.region_stride = static_cast<long long>(lt.row_region);
    dp.spr = static_cast<long long>(n - 1) * (per / 8);
    dp.total_stages = static_cast<long long>(cl_c) * dp.spr;
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
  const bool dl = (op == BCJR_OP_DENSE_BACKWARD_LAMBDA);
  const int N = n_seq > 0 ? n_seq : 1;
  int clusters = 0, parts = 0;
  if (dense_tc_clusters(adjoint, N, &clusters) != BCJR_OK) return 0;
  if (dl && dlam_parts(&parts) != BCJR_OK) return 0;
  const int chunk = dl ? clusters * bcjr::dense_tc_tile_seqs(adjoint) : N;
  return dense_tc_layout(adjoint, clusters, seq_len, chunk < N ? chunk : N, dl ? parts : 0).total;
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
