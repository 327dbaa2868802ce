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

#ifdef __cplusplus
}
#endif

#endif /* POLAR_ATTN_SELFTEST_H */
