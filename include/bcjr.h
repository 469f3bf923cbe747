/*
 * bcjr.h -- C ABI of libbcjr, a B200 (sm_100a) library for the hot path of
 * BCJR-QAT ("BCJR-QAT: A Differentiable Relaxation of Trellis-Coded Weight
 * Quantization", 2026): the temperature-T BCJR forward-backward over a
 * trellis, its soft codeword, the exact vector-Jacobian product of that
 * codeword, and the hard (T -> 0) Viterbi decode.
 *
 * Conventions shared by every call
 * --------------------------------
 *  - All array arguments are DEVICE pointers to row-major, contiguous, float32
 *    (or int32) buffers owned by the caller.  The library keeps no pointer
 *    after a call returns and allocates nothing on these paths: scratch comes
 *    from the caller's `workspace`, at least bcjr_workspace_size(...) bytes,
 *    256-byte aligned.  A workspace may be reused by later calls on the same
 *    stream; two calls in flight at once need two workspaces.
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL is the
 *    legacy default stream) and returns a bcjr_status.  Argument errors are
 *    found on the host before anything is launched and nothing is written.
 *    Errors the GPU finds (a non-finite log-partition function or metric)
 *    are OR-ed into a status word inside the workspace; read it with
 *    bcjr_get_status, which synchronises the stream.  No call aborts, throws
 *    or prints.
 *  - Trellis ("BCJR-QAT", technical summary, "core mechanism"; the bitshift
 *    structure is the standard trellis of trellis-coded quantization):
 *      S = 2^state_bits states, K = 2^k branches per state,
 *      pred(s) = { (j << (state_bits - k)) | (s >> k) : 0 <= j < K },
 *      emission log-weight phi_t(s) = -(w_t - codebook[s])^2 / T,
 *      uniform initial state, free final state.
 *    Supported here: 1 <= k <= 4, 2k <= state_bits <= 16.
 *  - Paths are weighted by exp(sum_t phi_t(s_t)) (Boltzmann weights at
 *    temperature T, "core mechanism"); the marginals are
 *    p_T(s_t = s | w) and the soft codeword is
 *      w_hat_t = sum_s codebook[s] p_T(s_t = s | w).
 */
#ifndef BCJR_H
#define BCJR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* bcjr_stream_t; /* same type as cudaStream_t */

typedef enum {
  BCJR_OK = 0,
  BCJR_ERR_INVALID_ARG = 1, /* null pointer, non-positive size, T <= 0 or not finite, misalignment */
  BCJR_ERR_UNSUPPORTED = 2, /* valid problem outside what the kernels cover (see limits above) */
  BCJR_ERR_WORKSPACE = 3,   /* workspace smaller than bcjr_workspace_size(...) */
  BCJR_ERR_CUDA = 4,        /* a CUDA runtime call or launch failed */
  BCJR_ERR_TIMEOUT = 5,     /* a bounded device-side wait gave up (reported through the status word) */
  BCJR_ERR_NONFINITE = 6    /* the device saw a NaN/inf log-partition function or path metric */
} bcjr_status;

/* Options; pass NULL for the defaults. */
typedef struct {
  /* Keep the forward group vector every C steps and recompute the others
   * during the backward sweep; 0 selects C = 1 (keep every step). */
  int checkpoint_interval;
  /* Sequences a thread-block-cluster team (state_bits >= 14) keeps in
   * flight, so that one sequence's exchange and barrier hide behind the
   * others' steps.  0 = automatic (two when k >= 2, one for k = 1).  2, 3 or 4
   * may be requested for bcjr_forward with k >= 2 (BCJR_ERR_UNSUPPORTED when
   * the buffers do not fit in shared memory), 2 for bcjr_backward; values
   * outside 0..4 are BCJR_ERR_INVALID_ARG.  Ignored by single-CTA teams; the
   * dense calls accept only 0. */
  int sequences_in_flight;
  /* Testing aid for the bounded device-side waits; 0 in normal use.  When
   * positive, a bcjr_forward / bcjr_backward call whose team is a
   * thread-block cluster (state_bits >= 14) runs, before any exchange between
   * the cluster's CTAs starts, one wait on an mbarrier that nothing arrives
   * at, bounded at this many SM clock cycles; the wait gives up, the call
   * computes nothing and bcjr_get_status then reports BCJR_ERR_TIMEOUT.  It
   * exercises the same bounded wait and status path as the exchange, with
   * nothing in flight.  Ignored by single-CTA teams and the other calls. */
  int timeout_probe_cycles;
  int reserved[5]; /* set to zero */
} bcjr_options;

typedef enum {
  BCJR_OP_FORWARD = 0,
  BCJR_OP_BACKWARD = 1,
  BCJR_OP_VITERBI = 2,
  BCJR_OP_DENSE_FORWARD = 3,
  BCJR_OP_DENSE_BACKWARD = 4,
  BCJR_OP_DENSE_BACKWARD_LAMBDA = 5
} bcjr_op;

/* Workspace bytes that a call of `op` with these sizes needs on the current
 * device.  For the dense ops, state_bits = log2(n_states) and k is ignored.
 * Returns 0 if the arguments are invalid or unsupported. */
size_t bcjr_workspace_size(int op, int state_bits, int k, int seq_len, int n_seq,
                           const bcjr_options* opt);

/*
 * Soft codeword ("core mechanism": w_hat_t = sum_s c(s) p_T(s_t = s | w)).
 *   w          [n_seq][seq_len]  weight preimages, one weight per step
 *   codebook   [S]               codeword of each state
 *   T          temperature > 0
 *   w_hat      [n_seq][seq_len]  out: soft codeword
 *   marginals  [n_seq][seq_len][S] out, or NULL: p_T(s_t = s | w)
 *   log_z      [n_seq] out, or NULL: natural log of sum over paths of exp(sum_t phi_t(s_t))
 *              (the 1/S of the uniform start is not included)
 */
bcjr_status bcjr_forward(const float* w, const float* codebook, float T, int state_bits, int k,
                         int seq_len, int n_seq, float* w_hat, float* marginals, float* log_z,
                         const bcjr_options* opt, void* workspace, size_t workspace_bytes,
                         bcjr_stream_t stream);

/*
 * bcjr_forward without a workspace argument: the same computation and outputs,
 * with scratch taken from a statically allocated device array of
 * BCJR_STATIC_SCRATCH_BYTES per device, so the call allocates no memory and
 * needs none from the caller.  The paper has no counterpart; this is a library
 * convenience for callers that cannot allocate device memory at call time.
 *  - The first call on each device looks up that device's copy of the array
 *    (which may load the library's module on it) and sets up the launch
 *    geometry; make that first call before any stream capture.  No claim is
 *    made about use inside a CUDA graph capture.
 *  - Returns BCJR_ERR_WORKSPACE, before launching anything, when the problem
 *    needs more than BCJR_STATIC_SCRATCH_BYTES, i.e. when
 *    bcjr_workspace_size(BCJR_OP_FORWARD, ...) is larger.
 *  - The device-side status word lives in the array and is cleared at the
 *    start of every call; read it with bcjr_static_scratch_status (below),
 *    which reports BCJR_ERR_TIMEOUT or BCJR_ERR_NONFINITE from the last call
 *    on the current device.
 *  - All calls on one device share the one array: two calls whose work
 *    overlaps in time (on different streams, or from several host threads
 *    without ordering) race on it and give wrong results.  Order them on one
 *    stream or with events.
 *  - Footprint: every device that loads the library holds the 32 MiB array
 *    until the process exits, whether or not it ever calls this entry point.
 *    With the CUDA runtime's default lazy module loading that happens on the
 *    first use of the library on the device; with CUDA_MODULE_LOADING=EAGER
 *    at context creation.
 *  - The address of the array is looked up once per device and cached for the
 *    life of the process; a device reset (cudaDeviceReset) invalidates it, so
 *    do not call this entry point on a device after resetting it.
 *  - The calls use the current device: make the device that holds the
 *    arguments current, and pass a stream of that device.
 */
#define BCJR_STATIC_SCRATCH_BYTES (32u << 20) /* 32 MiB */
bcjr_status bcjr_forward_static_scratch(const float* w, const float* codebook, float T, int state_bits,
                                        int k, int seq_len, int n_seq, float* w_hat, float* marginals,
                                        float* log_z, const bcjr_options* opt, bcjr_stream_t stream);

/* Synchronise `stream` and return the device-side status of the most recent
 * bcjr_forward_static_scratch call on the current device (BCJR_OK,
 * BCJR_ERR_NONFINITE or BCJR_ERR_TIMEOUT), the counterpart of bcjr_get_status
 * for the static scratch.  Allocates nothing. */
bcjr_status bcjr_static_scratch_status(bcjr_stream_t stream);

/*
 * Vector-Jacobian product of the soft codeword ("key technical innovations":
 * exact gradients through the trellis, differentiable in the weight preimage
 * and the trellis parameters).  With L = sum_t grad_w_hat_t w_hat_t:
 *   grad_w[n_seq][seq_len] = dL/dw
 *   grad_codebook[S]       = dL/dcodebook summed over all sequences
 *                            (added to the existing contents when
 *                            accumulate_codebook != 0, else overwritten)
 * w_hat is the soft codeword of the same (w, codebook, T); it is only used to
 * centre the accumulators, and the result does not depend on its exact value.
 */
bcjr_status bcjr_backward(const float* grad_w_hat, const float* w, const float* codebook,
                          const float* w_hat, float T, int state_bits, int k, int seq_len,
                          int n_seq, float* grad_w, float* grad_codebook, int accumulate_codebook,
                          const bcjr_options* opt, void* workspace, size_t workspace_bytes,
                          bcjr_stream_t stream);

/*
 * Hard decode, the T -> 0 limit ("core mechanism": the Viterbi argmax is the
 * zero-temperature limit of the Boltzmann distribution over paths): the path
 * minimising sum_t (w_t - codebook[s_t])^2, computed in float64 with ties to
 * the lowest predecessor index and the lowest final state.
 *   states  [n_seq][seq_len] out (int32)
 *   w_hard  [n_seq][seq_len] out, or NULL: codebook[states]
 */
bcjr_status viterbi_decode(const float* w, const float* codebook, int state_bits, int k,
                           int seq_len, int n_seq, int32_t* states, float* w_hard,
                           void* workspace, size_t workspace_bytes, bcjr_stream_t stream);

/*
 * Dense (fully connected) trellis: the transfer-matrix form of the abstract
 * (a 1D Ising-like chain).  Path log-weight sum_t phi_t(s_t) +
 * sum_{t>=1} log_trans[s_{t-1}][s_t]; log_trans is [n_states][n_states],
 * row = source state.  Same outputs and conventions as the bitshift calls.
 * Supported: n_states = 256.  Every step's forward vector is kept (no recompute
 * schedule), so checkpoint_interval must be 0 or 1; the workspace holds 32 KiB
 * per step per 128 sequences in flight for the forward call and 32 KiB per step
 * per 64 sequences in flight for the backward call (sequences in flight: up to
 * 128 x 33 and 64 x 33 on a B200).  The per-step contractions run on the
 * tensor cores in three-pass tf32 (float32-level accuracy).
 */
bcjr_status bcjr_dense_forward(const float* w, const float* codebook, const float* log_trans,
                               float T, int n_states, int seq_len, int n_seq, float* w_hat,
                               float* marginals, float* log_z, const bcjr_options* opt,
                               void* workspace, size_t workspace_bytes, bcjr_stream_t stream);
bcjr_status bcjr_dense_backward(const float* grad_w_hat, const float* w, const float* codebook,
                                const float* log_trans, const float* w_hat, float T, int n_states,
                                int seq_len, int n_seq, float* grad_w, float* grad_codebook,
                                int accumulate_codebook, const bcjr_options* opt, void* workspace,
                                size_t workspace_bytes, bcjr_stream_t stream);

/*
 * bcjr_dense_backward plus the gradient with respect to the log-transitions
 * ("key technical innovations": exact gradients with respect to the trellis
 * parameters).  Lambda[p][r] enters the path log-weight once per transition
 * p -> r, so with L = sum_t grad_w_hat_t w_hat_t and G = sum_t grad_w_hat_t c(s_t),
 *   grad_log_trans[p][r] = dL/dLambda[p][r] = Cov(G, number of transitions p -> r),
 * summed over all sequences.  grad_log_trans [n_states][n_states] is required
 * (row = source state); with accumulate != 0 both grad_codebook and
 * grad_log_trans are added to, otherwise overwritten.  The sum over
 * (sequence, transition) rows runs on the tensor cores in three-pass tf32
 * (float32-level accuracy).  Workspace: bcjr_workspace_size(BCJR_OP_DENSE_BACKWARD_LAMBDA, ...),
 * which adds four 64 KiB rows per step per 64 sequences in flight and a 256 KiB
 * partial sum per SM; batches longer than one 64-sequence tile per resident
 * cluster run in several launches inside the call.
 */
bcjr_status bcjr_dense_backward_lambda(const float* grad_w_hat, const float* w, const float* codebook,
                                       const float* log_trans, const float* w_hat, float T, int n_states,
                                       int seq_len, int n_seq, float* grad_w, float* grad_codebook,
                                       float* grad_log_trans, int accumulate, const bcjr_options* opt,
                                       void* workspace, size_t workspace_bytes, bcjr_stream_t stream);

/* Synchronise `stream` and return the device-side status of the most recent
 * call that used `workspace` (BCJR_OK, BCJR_ERR_NONFINITE or BCJR_ERR_TIMEOUT). */
bcjr_status bcjr_get_status(const void* workspace, bcjr_stream_t stream);

/* Static, human-readable name of a status code. */
const char* bcjr_status_string(bcjr_status status);

/* Library version as an integer (major * 10000 + minor * 100 + patch). */
int bcjr_version(void);

#ifdef __cplusplus
}
#endif

#endif /* BCJR_H */
