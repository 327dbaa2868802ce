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

/*
 * The paged decode with one query head per CTA: the same kernels, arguments,
 * layouts, results and errors as polar_attn_decode_paged, except that each
 * CTA reads the key/value pages of its query head's kv head for that head
 * alone, so that every page is read once per query head rather than once per
 * group.  It exists to measure the DRAM traffic the grouped kernel saves
 * ("GQA-Grouped Paged Decode Kernel", section 2.2: a group of Hq/Hkv query
 * heads shares each page read, cutting decode traffic by that factor).
 * Single-token decode only; workspace as polar_attn_decode_workspace_size.
 */
polar_status_t polar_attn_selftest_decode_per_head(const void *q, const void *kv_pages,
                                                   int num_pages, const int32_t *page_table,
                                                   int max_pages, const int32_t *seqlens,
                                                   int num_seqs, const float *u,
                                                   const polar_params_t *params, void *out,
                                                   float *neff_out, void *workspace,
                                                   size_t ws_bytes, void *stream);

/*
 * Host logic only (no device work): the row segments polar_attn_fwd_host uses
 * for the tensor-core prefill of T rows, in the order it sends them, from the
 * last rows to the first.  Segment i covers rows seg_lo[i] .. seg_hi[i] - 1;
 * about T/4 rows from the top, then halves down to 1024 rows, boundaries on
 * 128-row query tiles, one segment below T = 2048.  Writes at most `cap`
 * segments (the last always reaches row 0) and returns their number, or -1
 * for T < 0, cap < 1 or a NULL pointer.  Host pointers, owned by the caller.
 */
int polar_attn_selftest_fwd_host_segments(int T, int *seg_lo, int *seg_hi, int cap);

#ifdef __cplusplus
}
#endif

#endif /* POLAR_ATTN_SELFTEST_H */
