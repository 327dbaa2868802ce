// polar_internal.h -- host-side interface between the C ABI (api.cu) and the
// kernel launchers.  Not installed; not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace polar {

struct FwdLaunch {
    const void *q, *k, *v;
    const float *u;
    void *out;
    float *neff;  // may be null
    int B, T, Hq, Hkv;
    int dtype;    // POLAR_BF16 / POLAR_FP32
    float s, alpha, beta;
    int L;
    int window;   // 0: all causal keys; W > 0: the last W
    int *status;  // device status word
    float *moments;  // key-moment records (fwd_moments_bytes), or null
    float *state;    // training forward: saved row state (FwdState layout), or null
    int qt_lo, qt_cnt;  // query tiles qt_lo .. qt_lo + qt_cnt - 1 (qt_cnt 0: to the end)
    bool moments_ready;  // `moments` already holds the records of every key tile: no pre-pass
    cudaStream_t stream;
};

struct DecodeLaunch {
    const void *q, *kv_pages;
    int num_pages;
    const int32_t *page_table;
    int max_pages;
    const int32_t *seqlens;
    int num_seqs;
    const float *u;
    void *out;
    float *neff;
    int Hq, Hkv;
    float s, alpha, beta;
    int L;
    int window;  // 0: all cached positions; W > 0: the last W of each row's
    void *workspace;
    int chunk;  // query tokens per sequence (1 for plain decode)
    int per_head;  // test-only: one query head per CTA (pages read once per query head)
    int *status;
    cudaStream_t stream;
};

struct BwdLaunch {
    const void *q, *k, *v, *dout;  // dtype; dout like out
    const float *u;
    float *dq, *dk, *dv, *du;      // fp32 gradients, layouts of q, k, v, u
    int B, T, Hq, Hkv;
    int dtype;
    float s, alpha, beta;
    int L;
    int window;
    void *workspace;               // bwd_workspace_bytes
    int *status;                   // device status word
    cudaStream_t stream;
};

struct GdeltaLaunch {              // memory channel over whole sequences
    const void *q, *k, *v;         // [B, T, H, 64] dtype
    const float *alpha, *beta;     // [B, T, H]
    float *state;                  // [B, H, 64, 64], in place
    void *out;                     // [B, T, H, 64] dtype
    int B, T, H;
    int dtype, zero_init, accumulate;
    void *workspace;               // gdelta_workspace_bytes
    cudaStream_t stream;
};

struct GdeltaStepLaunch {          // one decode token per sequence, in place
    const void *q, *k, *v;         // [num_seqs, H, 64] dtype
    const float *alpha, *beta;     // [num_seqs, H]
    float *pool;                   // [num_slots, H, 64, 64]
    int num_slots;
    const int32_t *slots;          // [num_seqs]
    int num_seqs, H;
    int dtype, accumulate;
    void *out;                     // [num_seqs, H, 64] dtype
    int *status;
    cudaStream_t stream;
};

// Per-row coefficient record of the backward's bf16 path (fp32 words), written
// by the rows pass for every row of the sequence padded to a multiple of 128
// (rows past the end carry cl2 = c = 0 and nref = -inf, which give zero weights
// and zero dS without masks), read by the tensor-core dK/dV and dQ passes:
//   w  = 2^(cl2 S + nref)
//   dS = w (c <dA, v> + e1 + e2 w) + e3 S + e4   (+ cdm at the row's first argmax)
enum BwdCoef {
    kBcCl2 = 0, kBcNref = 1, kBcC = 2, kBcE1 = 3, kBcE2 = 4, kBcE3 = 5, kBcE4 = 6, kBcCdm = 7,
    kBcJmax = 8, kBcLo = 9, kBcGT = 10, kBwdCoefWords = 16
};

// Saved row state of a training forward (fp32 words per (batch, head, row),
// [B][Hq][T][kFwdStateWords]): the streaming sums l, l2 of the weights
// 2^(cl2 S - cl2) (the fixed reference), the max raw dot, the raw sums S1, S2,
// |acc| and the first argmax key (int32 bits).  The backward rebuilds each
// row's coefficient record and dA from it, out and dL/dout.
enum FwdState {
    kFsL = 0, kFsL2 = 1, kFsMax = 2, kFsS1 = 3, kFsS2 = 4, kFsNorm = 5, kFsArg = 6,
    kFwdStateWords = 8
};

// Launchers return cudaSuccess or the launch error.
cudaError_t launch_fwd_simt(const FwdLaunch &a);
cudaError_t launch_fwd_tc(const FwdLaunch &a);
cudaError_t launch_decode(const DecodeLaunch &a);
cudaError_t launch_bwd(const BwdLaunch &a);
size_t bwd_workspace_bytes(int B, int T, int Hq);
// The tensor-core dK/dV and dQ passes of the bf16 backward, given the rows
// pass's coefficient records coef [B][Hq][Tpad][kBwdCoefWords] and dA rounded
// to bf16, dab [B][Hq][Tpad][64] (Tpad = T rounded up to 128).
cudaError_t launch_bwd_tc(const BwdLaunch &l, const float *coef, const void *dab);
// The rows pass of the bf16 backward on the tensor cores (fwd_tc.cu): writes
// coef and dab as above.  cudaErrorNotSupported where it does not apply.
cudaError_t launch_bwd_rows_tc(const BwdLaunch &l, float *coef, void *dab, int Tpad);
// Whether the training forward saves its row state for this shape on the
// current device (bf16, an even group size, the fixed exponential reference,
// the kernel's register plan); where it does not, the training forward is the
// plain forward and the backward recomputes the rows.  Negative: CUDA error.
int fwd_state_supported(int dtype, int T, int Hq, int Hkv, float s, float alpha, int L,
                        int window);
// The training forward with the saved row state (a.state non-null); only
// where fwd_state_supported holds.
cudaError_t launch_fwd_train_tc(const FwdLaunch &a);
// The bf16 backward from a training forward's saved state: rows kernel (record,
// dA, du partials), the tensor-core dK/dV and dQ passes, du.
cudaError_t launch_bwd_from_state(const BwdLaunch &l, const void *out, const float *state);
cudaError_t launch_gdelta_prefill(const GdeltaLaunch &a);
cudaError_t launch_gdelta_step(const GdeltaStepLaunch &a);
size_t gdelta_workspace_bytes(int B, int T, int H);

// Key moments of causal prefill (fwd_moments.cu): one record of kMomFloats
// fp32 (the 64 x 64 key Gram, then the 64 key sums) per (batch, kv head, full
// key tile), running sums within chunks of kMomChunk tiles.
constexpr int kMomChunk = 8;
constexpr int kMomFloats = 64 * 64 + 64;
int fwd_moment_records(int T);
// Whether launch_fwd_tc would read key-moment records for this launch (and so
// run the pre-pass for its tiles unless they are ready).
bool fwd_tc_reads_moments(const FwdLaunch &a);
size_t fwd_moments_bytes(int B, int T, int Hkv);
// Computes the records rec_lo .. rec_hi - 1 (rounded out to whole chunks).
cudaError_t launch_fwd_moments(const void *k, int B, int T, int Hkv, float *rec, int rec_lo,
                               int rec_hi, cudaStream_t stream);

// Loads the decode kernels' code onto the current device now rather than at
// their first launch (lazy module loading).
cudaError_t decode_preload();

// Device address of the per-device status word on the current device, or null.
int *device_status_word();

// Decode work split: pages per split and the partial-state bytes it needs.
int decode_pages_per_split(int num_seqs, int max_pages, int Hkv);
size_t decode_partials_bytes(int num_seqs, int max_pages, int Hq, int Hkv, int chunk);

// Bookkeeping shared by the launchers.
void count_launches(int n);
CUresult encode_tiled(CUtensorMap *map, CUtensorMapDataType dtype, uint32_t rank, void *base,
                      const uint64_t *dims, const uint64_t *strides_bytes, const uint32_t *box,
                      CUtensorMapSwizzle swizzle);

}  // namespace polar
