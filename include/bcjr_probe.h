/*
 * bcjr_probe.h -- measurement aid of libbcjr: the throughput of the B200's
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

#ifdef __cplusplus
}
#endif

#endif /* BCJR_PROBE_H */
