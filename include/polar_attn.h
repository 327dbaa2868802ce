/*
 * polar_attn.h -- C ABI of the B200 (sm_100a) Polar Attention library.
 *
 * The library computes the Polar Attention mixing step of "ATMA: Length-
 * Invariant Language Modeling via Polar Attention and Gated-Delta Compression
 * Memory" (H. Akbar; gist.science technical summary, section 2.1 "Polar
 * Attention: A Three-Channel Decomposition"):
 *
 *     out = content + count
 *
 * The third stream, the recurrent gated-delta memory, has its own entry
 * points in polar_gdelta.h; they can add their read into an output written
 * here (out = content + count + memory).
 *
 * For query row i of head h with visible keys j < n (n = i + 1 in causal
 * prefill, n = seqlen in decode) and kv head g = h / (Hq / Hkv):
 *
 *   tau     = 1 + alpha * ln(n / L_train)  if n > L_train, else 1
 *   z_j     = logit_scale * tau * <q_i, k_j>
 *   p_j     = softmax_j(z)
 *   content = (sum_j p_j v_j) / |sum_j p_j v_j|          direction channel
 *   n_eff   = 1 / sum_j p_j^2  (= l^2 / l2)              participation ratio
 *   z0      = mean(z) + std(z) * sqrt(2 ln n)            null-floor logit
 *   gate    = 1 / (1 + exp(-beta * (max_j z_j - z0)))    detection confidence
 *   count   = gate * tanh(ln(n_eff) / ln(L_train)) * u_h magnitude channel
 *
 * std is the population standard deviation of the n visible logits, and the
 * null logit (whose value vector is zero) enters only the gate, not n_eff.
 *
 * Conventions for every entry point:
 *  - Pointers named *_h are host memory; every other tensor pointer is device
 *    memory on the current CUDA device.  The caller owns all memory; the
 *    library allocates nothing, neither device nor pinned memory.
 *  - Calls are asynchronous and ordered on `stream` (a cudaStream_t; NULL is
 *    the legacy default stream), except the *_host calls, which synchronise
 *    `stream` before they return.
 *  - Argument, shape and alignment errors are detected on the host and
 *    returned at once, and nothing is launched.  Errors found on the device
 *    (a page id out of range, a sequence length out of range, a wait that
 *    timed out) are recorded in a per-device status word that
 *    polar_attn_get_status() reads.  The kernel involved skips the offending
 *    work; it never traps.
 *  - Inputs q and k must be L2-normalised rows (the method normalises queries
 *    and keys, section 2.1 "Stability Mechanism"); the library does not check
 *    this.  head_dim must be 64.
 *  - All tensors are contiguous, with 16-byte aligned base pointers.
 */
#ifndef POLAR_ATTN_H
#define POLAR_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    POLAR_OK = 0,
    POLAR_ERR_INVALID_ARG = 1, /* bad pointer, shape, stride or parameter */
    POLAR_ERR_UNSUPPORTED = 2, /* valid but not built (e.g. head_dim != 64) */
    POLAR_ERR_WORKSPACE = 3,   /* workspace or staging buffer too small */
    POLAR_ERR_BAD_PAGE = 4,    /* device: page id outside [0, num_pages) */
    POLAR_ERR_TIMEOUT = 5,     /* device: a bounded wait ran out */
    POLAR_ERR_CUDA = 6,        /* a CUDA runtime call failed */
    POLAR_ERR_BAD_SEQLEN = 7,  /* device: seqlen outside [1, max_pages*64] */
    POLAR_ERR_BAD_SLOT = 8     /* device: memory state slot >= num_slots (polar_gdelta.h) */
} polar_status_t;

typedef enum { POLAR_BF16 = 0, POLAR_FP32 = 1 } polar_dtype_t;

/* Implementation choice for polar_attn_fwd. */
typedef enum {
    POLAR_IMPL_AUTO = 0,  /* tensor-core kernel for bf16, SIMT kernel for fp32 */
    POLAR_IMPL_SIMT = 1,  /* CUDA-core kernel: fp32 FFMA on the exact inputs */
    POLAR_IMPL_TC = 2     /* tcgen05/TMEM tensor-core kernel (bf16 only) */
} polar_impl_t;

typedef struct {
    int B;            /* batch (prefill); ignored by decode */
    int T;            /* sequence length (prefill); ignored by decode */
    int Hq, Hkv;      /* query heads, key/value heads; Hq % Hkv == 0, Hq/Hkv <= 8 */
    int head_dim;     /* must be 64 */
    int dtype;        /* polar_dtype_t of q, k, v, kv pages and out */
    float logit_scale;/* s: logits are s * tau * <q, k>; typical 8 */
    float alpha;      /* length-temperature slope; typical 0.3 */
    int L_train;      /* training length L_train >= 2; typical 2048 */
    float beta;       /* gate slope; typical 1.0 */
    int causal;       /* prefill: must be 1 (row i sees keys 0..i) */
    int impl;         /* polar_impl_t, prefill only */
    int window;       /* 0: every causal key; W > 0: sliding window, only the last W
                         visible keys (prefill i-W+1..i, decode seqlen-W..seqlen-1);
                         n, and with it the length temperature and the null floor,
                         is then the windowed count.  The pages' results section
                         names the window as an ablation. */
} polar_params_t;

/* Fills *p with the typical constants above for the given shape (window 0). */
void polar_attn_default_params(polar_params_t *p, int B, int T, int Hq, int Hkv, int dtype);

/*
 * Causal prefill: the fused Polar Attention step over a whole sequence
 * ("Fused Polar Attention Kernel", section 2.2: participation ratios computed
 * online with O(block) memory from streaming accumulators with squared
 * correction factors; no T x T score matrix is stored).
 *
 *  q         [B, T, Hq,  64] dtype, device
 *  k, v      [B, T, Hkv, 64] dtype, device
 *  u         [Hq, 64] float32, device: the per-head count vectors u_h
 *  params    shape and method constants (read on the host during the call)
 *  out       [B, T, Hq, 64] dtype, device: content + count
 *  neff_out  [B, Hq, T] float32, device: n_eff per row (may be NULL)
 *  stream    cudaStream_t the work is ordered on
 *
 * Needs no scratch memory: the raw logit sums of the null floor are summed
 * score by score inside the kernel.  Returns POLAR_OK once the work is
 * enqueued, or an argument error with nothing launched.  B = 0 or T = 0 is a
 * no-op.
 */
polar_status_t polar_attn_fwd(const void *q, const void *k, const void *v, const float *u,
                              const polar_params_t *params, void *out, float *neff_out,
                              void *stream);

/*
 * polar_attn_fwd with a caller-owned workspace, which makes long prefills
 * faster (the same rows up to rounding).
 *
 *  workspace device scratch of at least polar_attn_fwd_workspace_size()
 *            bytes, or NULL (then ws_bytes is ignored and the call is
 *            polar_attn_fwd).  With it, the raw logit sums of the null floor
 *            over the key tiles left of a query tile come from key moments
 *            (sum k, sum k k^T) that a pre-pass writes here, instead of from
 *            every score: the same quantities, computed with less work per
 *            score (used from 32 query tiles on; with a sliding window, for
 *            windows of at least 4096 keys, from differences of key-moment
 *            prefixes over the key tiles every row of a tile sees in full).
 *            Contents on entry are ignored; calls that share a workspace must
 *            not overlap.  A non-NULL workspace smaller than required returns
 *            POLAR_ERR_WORKSPACE.
 * Other arguments as polar_attn_fwd.
 */
size_t polar_attn_fwd_workspace_size(const polar_params_t *params);

polar_status_t polar_attn_fwd_ws(const void *q, const void *k, const void *v, const float *u,
                                 const polar_params_t *params, void *out, float *neff_out,
                                 void *workspace, size_t ws_bytes, void *stream);

/*
 * Backward of the causal prefill: the gradients of a loss L with respect to
 * q, k, v and u, given dout = dL/dout (the training use of the fused step).
 * Each row's forward state is recomputed, and the chain rule runs through
 * the direction (acc/|acc|), the participation ratio n_eff = l^2/l2, the
 * tanh-log magnitude, the gate on max logit - null floor, and the floor's mean
 * and spread.  The max contributes through its first index (a subgradient).
 * The window (params->window) is honoured; the key-moment workspace of
 * polar_attn_fwd_ws plays no part.
 *
 *  q, k, v, u  as polar_attn_fwd (dtype bf16 or fp32)
 *  dout       [B, T, Hq, 64] dtype, device
 *  dq         [B, T, Hq, 64] float32, device
 *  dk, dv     [B, T, Hkv, 64] float32, device (summed over the group's heads)
 *  du         [Hq, 64] float32, device (summed over batch and rows)
 *  workspace  device scratch of at least polar_attn_bwd_workspace_size() bytes
 *             (per-row coefficients); contents on entry are ignored
 *
 * bf16 inputs: the contractions run on the tensor cores (tcgen05, bf16
 * operands, fp32 accumulation), with the weights, dS and dA rounded to bf16 as
 * operands; fp32 inputs: the CUDA cores in fp32.  Deterministic: no atomics,
 * fixed summation orders.  B = 0 or T = 0 writes du = 0 and nothing else.
 */
size_t polar_attn_bwd_workspace_size(const polar_params_t *params);

polar_status_t polar_attn_bwd(const void *q, const void *k, const void *v, const float *u,
                              const void *dout, const polar_params_t *params, float *dq,
                              float *dk, float *dv, float *du, void *workspace, size_t ws_bytes,
                              void *stream);

/*
 * Training pair: a forward that also saves each row's streaming state, and a
 * backward that starts from that state instead of recomputing the forward
 * sweep.  The state is what the fused kernel already carries per row ("Fused
 * Polar Attention Kernel", section 2.2 of the technical summary: the streaming
 * sums l and l2, the max logit, the null floor's raw sums) plus |acc| and the
 * first argmax key; the backward of section 3's training use needs nothing
 * else besides out and dL/dout.
 *
 *  state  [B, Hq, T, 8] float32, device, 16-byte aligned, owned by the caller
 *         (polar_attn_fwd_state_size bytes): per row l, l2 (weights relative
 *         to the fixed reference c log2 e), max_j <q, k_j>, S1, S2, |acc|,
 *         the first argmax key (int32 bits), 0.
 *
 * polar_attn_fwd_train writes out and neff_out as polar_attn_fwd does (equal up
 * to rounding: it never uses the key moments) and the state.  Where the state
 * path does not apply -- fp32 inputs, an odd group size Hq/Hkv, a logit scale
 * times length temperature above 28/log2(e) (the fixed reference's range),
 * params->impl = POLAR_IMPL_SIMT -- it is exactly polar_attn_fwd and leaves
 * `state` untouched; polar_attn_bwd_from_state, given the same params, then
 * recomputes the rows as polar_attn_bwd does.  So the pair is valid for every
 * shape polar_attn_fwd accepts.
 *
 * polar_attn_bwd_from_state: arguments, outputs, workspace and errors as
 * polar_attn_bwd, plus out (the training forward's output, [B, T, Hq, 64]
 * dtype) and its state, both unchanged since that call with the same params
 * and inputs.  With the state it runs a rows kernel over (row, head) in place
 * of the forward sweep; the direction comes from out - count * u_h, so dA
 * carries out's bf16 rounding.  Asynchronous on `stream`.
 */
size_t polar_attn_fwd_state_size(const polar_params_t *params);

polar_status_t polar_attn_fwd_train(const void *q, const void *k, const void *v, const float *u,
                                    const polar_params_t *params, void *out, float *neff_out,
                                    float *state, void *stream);

polar_status_t polar_attn_bwd_from_state(const void *q, const void *k, const void *v,
                                         const float *u, const void *out, const float *state,
                                         const void *dout, const polar_params_t *params,
                                         float *dq, float *dk, float *dv, float *du,
                                         void *workspace, size_t ws_bytes, void *stream);

/* Bytes of device staging that polar_attn_fwd_host needs for this shape
 * (inputs, outputs and the workspace of polar_attn_fwd_ws). */
size_t polar_attn_fwd_staging_size(const polar_params_t *params);

/*
 * polar_attn_fwd on host buffers: copies q, k, v, u from host memory (pinned
 * memory gives full copy bandwidth) into `staging` (device memory owned by the
 * caller, at least polar_attn_fwd_staging_size bytes), runs the prefill
 * (polar_attn_fwd_ws with its workspace in the staging buffer), copies
 * out and n_eff back to host memory, and synchronises `stream`.  The work
 * goes batch by batch.  For the tensor-core prefill a batch's k and v go in
 * first and its key moments are formed; its queries then go in row segment
 * by row segment (about T/4 rows from the top, then halves down to 1024 rows;
 * one segment below T = 2048), from the LAST rows to the first, so that the
 * longest causal rows start first and the call ends on the lightest segment.
 * Each segment's prefill starts as soon as its queries are in, alternating
 * between `stream` and a second compute stream, and its output rows are
 * copied back as soon as it is done (a batch's n_eff in one copy after its
 * last segment).  The copies run on two copy streams; the library
 * creates these three streams once per device and joins them to `stream`
 * through events.  The CUDA-core prefill goes whole batch by whole batch.  The
 * results are those of polar_attn_fwd_ws, bit for bit.  Host-buffer calls on
 * one device are serialised.  Argument errors return before anything is
 * queued; after a POLAR_ERR_CUDA return, copies or prefills already queued on
 * the library's streams may still run, so synchronise the device before the
 * staging buffer or the host buffers are reused.
 */
polar_status_t polar_attn_fwd_host(const void *q_h, const void *k_h, const void *v_h,
                                   const float *u_h, const polar_params_t *params, void *out_h,
                                   float *neff_h, void *staging, size_t staging_bytes,
                                   void *stream);

/*
 * Paged GQA decode: one query token per sequence against a paged KV cache
 * ("GQA-Grouped Paged Decode Kernel", section 2.2: decode reads the paged KV
 * cache blocks directly, and each key/value page is read once for all the
 * query heads of its group).
 *
 *  q          [num_seqs, Hq, 64] dtype, device
 *  kv_pages   [num_pages, 2, Hkv, 64, 64] dtype, device: page p holds 64
 *             tokens; [p][0] are keys and [p][1] values, head-major, so each
 *             (page, K|V, head) is one contiguous 64 x 64 block
 *  page_table [num_seqs, max_pages] int32, device: logical page -> physical
 *             page; entries at or past ceil(seqlen/64) are never read
 *  seqlens    [num_seqs] int32, device: tokens in the cache of each sequence,
 *             1 <= seqlen <= 64 * max_pages; the query sees all of them (its
 *             own key and value must already be in the cache)
 *  u          [Hq, 64] float32, device
 *  out        [num_seqs, Hq, 64] dtype, device
 *  neff_out   [num_seqs, Hq] float32, device (may be NULL)
 *  workspace  device scratch of at least polar_attn_decode_workspace_size()
 *             bytes for the per-split partial states; contents on entry are
 *             ignored.  Calls that share a workspace must not overlap.
 *
 * A page id outside [0, num_pages) sets POLAR_ERR_BAD_PAGE and that page is
 * skipped; a seqlen out of range sets POLAR_ERR_BAD_SEQLEN and that sequence
 * is skipped (its outputs are left unwritten).
 */
size_t polar_attn_decode_workspace_size(int num_seqs, int max_pages, const polar_params_t *params);

polar_status_t polar_attn_decode_paged(const void *q, const void *kv_pages, int num_pages,
                                       const int32_t *page_table, int max_pages,
                                       const int32_t *seqlens, int num_seqs, const float *u,
                                       const polar_params_t *params, void *out, float *neff_out,
                                       void *workspace, size_t ws_bytes, void *stream);

/*
 * Multi-token paged decode: `chunk` query tokens per sequence, for speculative
 * verification or chunked prefill against the paged cache (the pages'
 * evaluation decodes against 256K-token caches; this extends the grouped
 * decode of section 2.2 to several queries per sequence).
 *
 *  q        [num_seqs, chunk, Hq, 64] dtype, device: token t of sequence s is
 *           the query at cache position seqlen[s] - chunk + t (the chunk's own
 *           keys and values must already be in the cache)
 *  out      [num_seqs, chunk, Hq, 64] dtype, device
 *  neff_out [num_seqs, chunk, Hq] float32, device (may be NULL)
 *  other arguments as polar_attn_decode_paged.
 *
 * Token t sees the cache positions below n_t = seqlen - chunk + t + 1 (causal
 * within the chunk), with the length temperature of n_t; each token's row
 * equals polar_attn_decode_paged with seqlen n_t.  Every key/value page is read
 * once for all chunk x (Hq/Hkv) queries of its group.  Requires chunk >= 1,
 * (Hq/Hkv) * chunk <= 16 (else POLAR_ERR_UNSUPPORTED) and chunk <= seqlen <=
 * 64 * max_pages per sequence (else POLAR_ERR_BAD_SEQLEN on the device, and the
 * sequence is skipped).  chunk = 1 is polar_attn_decode_paged.
 */
size_t polar_attn_decode_chunk_workspace_size(int num_seqs, int max_pages, int chunk,
                                              const polar_params_t *params);

polar_status_t polar_attn_decode_paged_chunk(const void *q, const void *kv_pages, int num_pages,
                                             const int32_t *page_table, int max_pages,
                                             const int32_t *seqlens, int num_seqs, int chunk,
                                             const float *u, const polar_params_t *params,
                                             void *out, float *neff_out, void *workspace,
                                             size_t ws_bytes, void *stream);

/* Bytes of device staging that polar_attn_decode_paged_host needs. */
size_t polar_attn_decode_staging_size(int num_seqs, int max_pages, const polar_params_t *params);

/*
 * polar_attn_decode_paged with the per-step inputs (q, page_table, seqlens,
 * u) in host memory and the outputs returned to host memory; the KV pool stays
 * resident on the device.  Uses `staging` (device, caller-owned, at least
 * polar_attn_decode_staging_size bytes, which includes the workspace) and
 * synchronises `stream` before returning.
 */
polar_status_t polar_attn_decode_paged_host(const void *q_h, const void *kv_pages, int num_pages,
                                            const int32_t *page_table_h, int max_pages,
                                            const int32_t *seqlens_h, int num_seqs,
                                            const float *u_h, const polar_params_t *params,
                                            void *out_h, float *neff_h, void *staging,
                                            size_t staging_bytes, void *stream);

/*
 * Paged GQA decode for callers that cannot allocate device memory -- for
 * example a serving process that handed all free device memory to its KV-cache
 * pool at start-up, or a plug-in whose host framework gives it no device
 * allocator -- and so have no workspace to pass.  The paper has no counterpart;
 * this is a property of the library, not of the method.
 *
 * Same arguments, layouts, results and error reporting as
 * polar_attn_decode_paged, without the workspace: the per-split scratch lives
 * in a fixed array of POLAR_NOALLOC_SCRATCH_BYTES bytes of device memory that
 * the library holds on every device that loads it, until the process exits.
 * The call itself allocates nothing and calls no allocating routine.
 *  - A shape whose scratch (polar_attn_decode_workspace_size) exceeds
 *    POLAR_NOALLOC_SCRATCH_BYTES is rejected with POLAR_ERR_WORKSPACE and
 *    nothing is launched.
 *  - The first call on a device sets the device up, with that device current:
 *    it looks up the array's device address (a synchronous runtime query) and
 *    loads the library's decode kernels and status word onto the device.
 *    Under CUDA's lazy module loading (the default) that is when the array's
 *    POLAR_NOALLOC_SCRATCH_BYTES and the kernels' code take device memory, so
 *    make this first call before handing the remaining free memory to a pool,
 *    and before any stream capture.  A call with num_seqs = 0 (and otherwise
 *    valid arguments) does the set-up and nothing else; later calls take no
 *    device memory.
 *  - The addresses are kept for the life of the process: do not use the
 *    library across a device reset (cudaDeviceReset) on that device.
 *  - Every call on a device shares the one array and leaves its contents
 *    behind.  Nothing in it has to start at zero: each split writes its whole
 *    partial state before the merge reads it.  Calls whose work overlaps on the
 *    GPU (concurrent streams, or other host threads) race on the array; order
 *    them on one stream or serialise them.
 */
#define POLAR_NOALLOC_SCRATCH_BYTES (16u << 20)

polar_status_t polar_attn_decode_paged_noalloc(const void *q, const void *kv_pages,
                                               int num_pages, const int32_t *page_table,
                                               int max_pages, const int32_t *seqlens,
                                               int num_seqs, const float *u,
                                               const polar_params_t *params, void *out,
                                               float *neff_out, void *stream);

/*
 * Synchronises `stream`, returns the first device-side error recorded on the
 * current device since the last call (POLAR_OK if none) and clears it.
 */
polar_status_t polar_attn_get_status(void *stream);

/* Static English description of a status code. */
const char *polar_attn_status_string(polar_status_t status);

/* Number of kernel launches the library has enqueued on this process so far. */
uint64_t polar_attn_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* POLAR_ATTN_H */
