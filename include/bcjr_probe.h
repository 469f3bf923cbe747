/*
 * bcjr_probe.h -- measurement aids of libbcjr.  The throughput of the B200's
 * special-function (XU) pipe, which executes the 2^x and log2 instructions
 * that bound the BCJR forward-backward ("BCJR-QAT", technical summary, "key
 * technical innovations": the fused kernel's work is gather, log-sum-exp and
 * add, i.e. one exponential per trellis state and sweep).  The exp-pipe
 * roofline of the benchmark divides by this pipe's peak; the probe measures
 * that peak on the device at hand instead of taking it from a table.
 */
#ifndef BCJR_PROBE_H
#define BCJR_PROBE_H

#include <stdint.h>

#include "bcjr.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { BCJR_PROBE_EX2 = 0, BCJR_PROBE_LG2 = 1 } bcjr_probe_op;

/*
 * Launch one CTA of 1024 threads per SM; every thread runs 16 independent
 * chains of `iters` dependent ex2.approx.ftz.f32 (op = BCJR_PROBE_EX2) or
 * lg2.approx.ftz.f32 (op = BCJR_PROBE_LG2) instructions.  Each CTA counts its
 * own SM clock cycles between two CTA barriers around the chains, so
 *   ops per clock per SM = 1024 * 16 * iters / cycles[cta]
 * independently of the clock frequency.
 *   iters       >= 1, at most 1 << 20
 *   sink        [n_sm * 1024] floats, device: the chains' results (kept so
 *               that the compiler cannot drop them)
 *   cycles      [n_sm] int64, device: cycles counted by each CTA
 *   n_sm        number of CTAs launched, 1 .. 4096 (pass the SM count)
 * Asynchronous on `stream`; returns BCJR_ERR_INVALID_ARG for bad sizes or null
 * pointers and BCJR_ERR_CUDA if the launch fails.
 */
bcjr_status bcjr_probe_xu(int op, int iters, float* sink, long long* cycles, int n_sm,
                          bcjr_stream_t stream);

/*
 * The two costs that bound a step of the dense trellis's tensor-core kernels
 * (the transfer-matrix contraction of the abstract's 1D Ising-like chain).
 *
 * bcjr_probe_mma_tf32: one CTA of 128 threads per SM; one thread issues
 * `iters` tcgen05.mma.cta_group::1.kind::tf32 products with M = 128, K = 8
 * and the given N (16, 32, 64, 128 or 256), operand A read from tensor memory
 * and B from shared memory, into one tensor-memory accumulator, then waits
 * (bounded) for their completion.  cycles[cta] = SM clock cycles from the first
 * issue to the completion, so
 *   cycles per product = cycles[cta] / iters,
 *   MAC per clock per SM = 128 * N * 8 * iters / cycles[cta].
 *   iters   1 .. 1 << 20
 *   cycles  [n_sm] int64, device
 *   status  one int, device, zeroed by the caller: BCJR_ERR_TIMEOUT's bit is
 *           set if the wait ran out
 *   n_sm    CTAs launched, 1 .. 4096 (pass the SM count)
 *
 * bcjr_probe_dsmem: 4-CTA thread-block clusters of 256 threads; per round
 * every CTA stores reps x 32 KiB into each of the other three CTAs' shared
 * memory with st.async (completing on the receiver's mbarrier) and waits
 * (bounded) for the 3 x reps x 32 KiB it receives.  cycles[cta] = SM clock
 * cycles of all `rounds`, so bytes out per clock per SM =
 * 3 * 32768 * reps * rounds / cycles[cta].
 *   reps        1 .. 8
 *   rounds      1 .. 65536
 *   cycles      [4 * n_clusters] int64, device
 *   status      as above
 *   n_clusters  clusters launched, 1 .. 1024 (clusters beyond those that fit
 *               at once run later and measure the same)
 * bcjr_probe_dsmem_bulk: the same exchange (sizes, rounds, cycles) moved by
 * the bulk-copy engine instead of per-thread stores: every warp owns 4 KiB of
 * each 32 KiB slot and issues one cp.async.bulk from a local shared-memory
 * source into the peer's slot per `chunk_bytes` (a power of two, 128 .. 4096),
 * completing on the receiver's mbarrier.
 *
 * All three are asynchronous on `stream`; they return BCJR_ERR_INVALID_ARG for
 * bad sizes or null pointers and BCJR_ERR_CUDA if the launch fails.
 */
bcjr_status bcjr_probe_mma_tf32(int n, int iters, long long* cycles, int* status, int n_sm,
                                bcjr_stream_t stream);
bcjr_status bcjr_probe_dsmem(int reps, int rounds, long long* cycles, int* status, int n_clusters,
                             bcjr_stream_t stream);
bcjr_status bcjr_probe_dsmem_bulk(int chunk_bytes, int reps, int rounds, long long* cycles, int* status,
                                  int n_clusters, bcjr_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* BCJR_PROBE_H */
