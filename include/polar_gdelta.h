/*
 * polar_gdelta.h -- C ABI of the recurrent memory channel: the gated-delta
 * associative memory that ATMA adds as the third stream of a Polar Attention
 * layer ("ATMA: Length-Invariant Language Modeling via Polar Attention and
 * Gated-Delta Compression Memory", gist.science technical summary, section
 * 2.1 "Recurrent Memory Channel"; section 2.2 "In-Place Gated-Delta Step
 * Kernel").
 *
 *     out = content + count + memory
 *
 * The pages name the rule (gated delta, derived from Gated DeltaNet) and its
 * stability mechanism (L2-normalised keys and queries) but print no formula;
 * the library computes the published gated delta rule.  Per (sequence, head),
 * with the state S (64 x 64 fp32, row = value dimension, column = key
 * dimension) and token t:
 *
 *   qh    = q_t / |q_t| ,  kh = k_t / |k_t|   (computed here; a zero row stays 0)
 *   S_t   = alpha_t * S_{t-1} * (I - beta_t kh kh^T) + beta_t v_t kh^T
 *   o_t   = S_t qh                              (read after the write)
 *
 * alpha_t (decay gate) and beta_t (write strength) are per (token, head)
 * inputs in [0, 1]; values outside that range are computed as given, without
 * the stability guarantee.
 *
 * Conventions as in polar_attn.h: device pointers on the current device, the
 * caller owns all memory, calls are asynchronous on `stream`, host-detected
 * errors return at once with nothing launched, device-detected errors go to
 * the status word that polar_attn_get_status() reads.  Base pointers 16-byte
 * aligned; tensors contiguous.
 */
#ifndef POLAR_GDELTA_H
#define POLAR_GDELTA_H

#include <stddef.h>
#include <stdint.h>

#include "polar_attn.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct {
    int B;          /* sequences (prefill) */
    int T;          /* tokens per sequence (prefill) */
    int H;          /* memory heads */
    int head_dim;   /* must be 64 (key and value dimensions) */
    int dtype;      /* polar_dtype_t of q, k, v and out */
    int zero_init;  /* 1: the initial state is zero and `state` is not read
                       (prefill); 0: `state` holds S_0 */
    int accumulate; /* 0: out = o; 1: out += o (adds the memory stream into an
                       attention output, the pages' additive third stream) */
} polar_gdelta_params_t;

/*
 * Memory channel over whole sequences (prefill / training forward).
 *
 *  q, k, v    [B, T, H, 64] dtype (bf16 or fp32), device
 *  alpha      [B, T, H] float32, device
 *  beta       [B, T, H] float32, device
 *  state      [B, H, 64, 64] float32, device, in place: S_0 on entry (unless
 *             zero_init), the state after token T-1 on return
 *  out        [B, T, H, 64] dtype, device
 *  workspace  device scratch of at least polar_gdelta_prefill_workspace_size()
 *             bytes; contents on entry are ignored; calls sharing a
 *             workspace must not overlap.
 *
 * Computed chunk-parallel: tokens in chunks of 64; within a chunk the writes
 * are solved at once (a unit lower-triangular system over the chunk's keys),
 * and the state passes from chunk to chunk, all in fp32.  With few (sequence,
 * head) pairs and many chunks (bf16), the chunks also go in groups: each
 * group's effect on the state is the affine map S -> S M + E, the groups'
 * initial states follow from those maps in sequence, and the groups then run
 * side by side.  The result equals the token-by-token recurrence up to fp32
 * rounding.  alpha below 1.6e-38 acts
 * as 1.6e-38.  B = 0 or T = 0 leaves everything unchanged.
 */
size_t polar_gdelta_prefill_workspace_size(const polar_gdelta_params_t *params);

polar_status_t polar_gdelta_prefill(const void *q, const void *k, const void *v,
                                    const float *alpha, const float *beta, float *state,
                                    const polar_gdelta_params_t *params, void *out,
                                    void *workspace, size_t ws_bytes, void *stream);

/*
 * One decode token per sequence, updating each sequence's state in place in a
 * pool of state slots (section 2.2: the step reads and writes the memory where
 * it lives, with no gather into a batch buffer and scatter back).
 *
 *  q, k, v     [num_seqs, H, 64] dtype (bf16 or fp32), device
 *  alpha, beta [num_seqs, H] float32, device
 *  state_pool  [num_slots, H, 64, 64] float32, device: slot s holds the states
 *              of one sequence's H heads
 *  slots       [num_seqs] int32, device: the slot of each sequence; a negative slot skips
 *              the sequence (nothing read or written).  Slots of one call must
 *              be distinct.  A slot >= num_slots sets POLAR_ERR_BAD_SLOT and
 *              the sequence is skipped.
 *  out         [num_seqs, H, 64] dtype, device (params->accumulate as above)
 *
 * params->B and params->T are ignored.
 */
polar_status_t polar_gdelta_step(const void *q, const void *k, const void *v,
                                 const float *alpha, const float *beta, float *state_pool,
                                 int num_slots, const int32_t *slots, int num_seqs,
                                 const polar_gdelta_params_t *params, void *out, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* POLAR_GDELTA_H */
