/*
 * polar_attn_selftest.h -- device self-tests of building blocks that the
 * kernels use, exported so that the test-suite can check them on a GPU.  Not
 * part of the computation's ABI; the paper has no counterpart.
 */
#ifndef POLAR_ATTN_SELFTEST_H
#define POLAR_ATTN_SELFTEST_H

#include "polar_attn.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Evaluates, for each of the n device floats x[i] (n even, -126 < x < 128),
 * the prefill kernel's FMA-pipe exponential 2^x (Cody-Waite reduction and a
 * degree-4 minimax polynomial) into poly[i], and the MUFU ex2.approx result
 * into mufu[i].  Asynchronous on `stream`; device pointers, 8-byte aligned.
 */
polar_status_t polar_attn_selftest_exp2(const float *x, float *poly, float *mufu, int n,
                                        void *stream);

/*
 * Failure detection: launches one CTA whose single mbarrier wait can never
 * complete (nothing arrives on the barrier).  The wait is the kernels' own
 * bounded wait: after its cycle budget (about a second) it records
 * POLAR_ERR_TIMEOUT in the device status word and the kernel exits normally,
 * so polar_attn_get_status then returns POLAR_ERR_TIMEOUT and the context
 * stays usable.  Asynchronous on `stream`.
 */
polar_status_t polar_attn_selftest_timeout(void *stream);

#ifdef __cplusplus
}
#endif

#endif /* POLAR_ATTN_SELFTEST_H */
