// fwd_tc.cu -- tcgen05/TMEM tensor-core causal Polar Attention prefill (sm_100a).
//
// "Fused Polar Attention Kernel" (ATMA technical summary, section 2.2): the
// participation ratio is computed online with O(block) memory, from streaming
// accumulators rescaled by squared correction factors, and the T x T score
// matrix is never stored.  The two dense contractions of the step, S = Q K^T
// and O += P V, run on the 5th-generation tensor cores with fp32 accumulators
// in tensor memory; everything between them (length temperature, running max,
// l, l2, the raw-dot sums of the null floor, the bf16 P tile) runs in the
// softmax warpgroups, one query row per thread.
//
// CTA work unit: two query heads of one key/value group over the same 128
// query rows, so both heads share every K/V tile and have the same causal
// extent.  Warp roles:
//   warp 0      TMA producer: Q tiles once, then K/V tiles into a 4-stage ring
//   warp 1      tensor-memory allocator and the score-MMA issuer (one thread)
//   warp 2      the PV-MMA issuer (one thread)
//   warp 3      key moments of the keys left of the query tile (kMoments), else idle
//   softmax     one warpgroup per head slot (warps 4-7, 8-11; TMEM lanes 0-127),
//               or with split rows two per head slot (warps 4-11 for slot 0, the
//               first four on keys 0-63 of each tile, the next four on 64-127;
//               warps 12-19 for slot 1)
// Tensor memory (512 columns): S0 S1 (128 fp32 columns each), P0 P1 (128 bf16
// packed in 64 columns each), O0 O1 (64 fp32 columns each).
// Two issuing threads keep the tensor core fed: one issues S_i(j) as soon as
// softmax i has copied S_i(j-1) out of tensor memory (barrier s_free), the
// other PV_i(j) as soon as P_i(j) is in tensor memory (p_full), so neither
// waits behind the other's queue.  A commit after PV_i(j) (pv_done) tells
// softmax i that P_i may be overwritten and that O_i is current, so it can
// rescale O_i in place before it releases P_i(j+1).
#include <algorithm>
#include <atomic>

#include "bwd_coef.cuh"
#include "polar_attn_selftest.h"
#include "polar_common.cuh"
#include "polar_internal.h"
#include "tc_common.cuh"

namespace polar {
namespace {

constexpr int kBM = 128;               // query rows per head slot
constexpr int kBN = 128;               // keys per tile
constexpr int kStagesKV = 4;           // K/V ring depth
constexpr int kTileBytes = 128 * 128;  // 128 rows x 64 bf16
constexpr int kGramBytes = 64 * 128;   // 64 x 64 bf16, 128B-swizzled, K-major
// The key moments pay off from this many query tiles on: below it the
// pre-pass and the per-CTA moment epilogue cost more than they save.
constexpr int kMomMinTiles = 32;
constexpr int kSmemBytes = (2 + 2 * kStagesKV) * kTileBytes + 2 * kGramBytes + 256 + 1024;

// Tensor-memory column map.
constexpr uint32_t kColS0 = 0, kColS1 = 128, kColP0 = 256, kColP1 = 320, kColO0 = 384,
                   kColO1 = 448;

// 2^x on the FMA pipe for two values at once (Cody-Waite range reduction and a
// degree-4 minimax polynomial; the FlashAttention-4 write-up publishes the
// idea of sharing the exponentials between this and the MUFU unit).  x = n + f
// with n = round(x), f in [-1/2, 1/2]; p(f) ~ 2^f with relative error below
// 4e-6 in fp32 (coefficients from exp2_poly_coeffs.py, which derives them by
// a Remez exchange); 2^n enters as an integer add to the exponent field.
// Valid for -126 < x < 128; callers guarantee the range.
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
    constexpr float kShift = 12582912.0f;  // 1.5 * 2^23: x + kShift rounds x to an integer
    const float2 j = f2_add(x, make_float2(kShift, kShift));
    const float2 r = f2_add(j, make_float2(-kShift, -kShift));
    const float2 f = f2_fma(r, make_float2(-1.f, -1.f), x);
    float2 p = make_float2(9.570102207e-03f, 9.570102207e-03f);
    p = f2_fma(p, f, make_float2(5.591785908e-02f, 5.591785908e-02f));
    p = f2_fma(p, f, make_float2(2.402474433e-01f, 2.402474433e-01f));
    p = f2_fma(p, f, make_float2(6.931217909e-01f, 6.931217909e-01f));
    p = f2_fma(p, f, make_float2(1.0f, 1.0f));
    const uint32_t px = __float_as_uint(p.x) + (__float_as_uint(j.x) << 23);
    const uint32_t py = __float_as_uint(p.y) + (__float_as_uint(j.y) << 23);
    return make_float2(__uint_as_float(px), __uint_as_float(py));
}


#ifndef POLAR_TC_SPLIT_POLY_MASK
// The same for the half-row pass of the split softmax (16 pairs per chunk):
// 0x0101 = 2 of 16, the best of the measured shares on B200.
#define POLAR_TC_SPLIT_POLY_MASK 0x0101
#endif

#ifndef POLAR_TC_POLY_MASK
// Which of every 16 exponential pairs of a full tile go to the polynomial
// (bit e set: pair e); the rest use MUFU ex2.  0x0202 = 2 of 16.
#define POLAR_TC_POLY_MASK 0x0202
#endif

// Row statistics of one 128-key tile of S (raw dots, one row per thread):
// max, sum and sum of squares over the visible keys.  Independent partial
// accumulators keep the dependency chains short.  kDiag: some keys of the
// tile are invisible to the row (key e is visible iff tlo <= e <= thi: after
// the row's own position, or before its sliding window); they are set to -inf
// in sr.
template <bool kDiag>
__device__ __forceinline__ void row_stats(uint32_t (&sr)[4][32], int thi, int tlo, float &tmax,
                                          float &ts1, float &ts2) {
    if (!kDiag) {
        float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        float2 a1[4], a2[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) a1[q] = a2[q] = make_float2(0.f, 0.f);
#pragma unroll
        for (int e = 0; e < 64; ++e) {
            const float x0 = __uint_as_float(sr[e >> 4][2 * (e & 15)]);
            const float x1 = __uint_as_float(sr[e >> 4][2 * (e & 15) + 1]);
            mx[e & 3] = max3(mx[e & 3], x0, x1);
            const float2 v = make_float2(x0, x1);
            a1[e & 3] = f2_add(a1[e & 3], v);
            a2[e & 3] = f2_fma(v, v, a2[e & 3]);
        }
        tmax = fmaxf(max3(mx[0], mx[1], mx[2]), mx[3]);
        const float2 b1 = f2_add(f2_add(a1[0], a1[1]), f2_add(a1[2], a1[3]));
        const float2 b2 = f2_add(f2_add(a2[0], a2[1]), f2_add(a2[2], a2[3]));
        ts1 = b1.x + b1.y;
        ts2 = b2.x + b2.y;
    } else {
        float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        float a1[4] = {0.f, 0.f, 0.f, 0.f}, a2[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int e = 0; e < 128; ++e) {
            const bool vis = e <= thi && e >= tlo;
            const float x = __uint_as_float(sr[e >> 5][e & 31]);
            const float xv = vis ? x : 0.f;
            sr[e >> 5][e & 31] = __float_as_uint(vis ? x : -INFINITY);
            mx[e & 3] = fmaxf(mx[e & 3], vis ? x : -INFINITY);
            a1[e & 3] += xv;
            a2[e & 3] = fmaf(xv, xv, a2[e & 3]);
        }
        tmax = fmaxf(max3(mx[0], mx[1], mx[2]), mx[3]);
        ts1 = (a1[0] + a1[1]) + (a1[2] + a1[3]);
        ts2 = (a2[0] + a2[1]) + (a2[2] + a2[3]);
    }
}

// Weights p = 2^(c*log2e*S - m_ref) of one tile: their sum and sum of squares
// (for l and l2), and the bf16 pairs of the P tile in pk.
// kPoly: the pairs selected by POLAR_TC_POLY_MASK use the FMA-pipe polynomial
// (full tiles only; the diagonal tile's -inf entries use ex2, which gives 0).
template <bool kPoly>
__device__ __forceinline__ void row_weights(const uint32_t (&sr)[4][32], float2 sc2, float neg_m,
                                            uint32_t (&pk)[4][16], float &tl, float &tl2) {
    const float2 nm = make_float2(neg_m, neg_m);
    float2 la[2], l2a[2];
    la[0] = la[1] = l2a[0] = l2a[1] = make_float2(0.f, 0.f);
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const float2 sv = make_float2(__uint_as_float(sr[cc][2 * e]),
                                          __uint_as_float(sr[cc][2 * e + 1]));
            const float2 x = f2_fma(sv, sc2, nm);
            float2 p;
            if (kPoly && ((POLAR_TC_POLY_MASK >> e) & 1)) {
                p = exp2_poly2(make_float2(fmaxf(x.x, -126.f), fmaxf(x.y, -126.f)));
            } else {
                p.x = ex2(x.x);
                p.y = ex2(x.y);
            }
            la[e & 1] = f2_add(la[e & 1], p);
            l2a[e & 1] = f2_fma(p, p, l2a[e & 1]);
            pk[cc][e] = pack_bf16(p.x, p.y);
        }
    }
    const float2 sl = f2_add(la[0], la[1]), sl2 = f2_add(l2a[0], l2a[1]);
    tl = sl.x + sl.y;
    tl2 = sl2.x + sl2.y;
}

// One pass over a tile with a fixed exponential reference (see the kernel's
// kFixedRef): the weights p = 2^(c*log2e*S + neg_m) are computed at once, with
// no wait for the tile max, and returned packed as bf16 pairs in pk; the max,
// sum and sum of squares of the raw dots (for the gate and the null floor) and
// the sums of p and p^2 (l, l2) accumulate alongside.  kDiag masks the keys
// outside tlo .. thi (after the row's own position or before its sliding
// window: p = 0, excluded from every sum).
template <bool kDiag, bool kPoly>
__device__ __forceinline__ void fused_tile(const uint32_t (&sr)[4][32], int thi, int tlo,
                                           float2 sc2, float neg_m, uint32_t (&pk)[4][16],
                                           float &tmax, float &ts1, float &ts2, float &tl,
                                           float &tl2) {
    const float2 nm = make_float2(neg_m, neg_m);
    float mx[2] = {-INFINITY, -INFINITY};
    float2 a1 = make_float2(0.f, 0.f), a2 = a1, la = a1, l2a = a1;
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            float2 sv = make_float2(__uint_as_float(sr[cc][2 * e]), __uint_as_float(sr[cc][2 * e + 1]));
            float2 x;
            if (kDiag) {
                const int col = 32 * cc + 2 * e;
                const bool v0 = col <= thi && col >= tlo, v1 = col + 1 <= thi && col + 1 >= tlo;
                mx[e & 1] = max3(mx[e & 1], v0 ? sv.x : -INFINITY, v1 ? sv.y : -INFINITY);
                x = f2_fma(sv, sc2, nm);
                x.x = v0 ? x.x : -INFINITY;
                x.y = v1 ? x.y : -INFINITY;
                sv.x = v0 ? sv.x : 0.f;
                sv.y = v1 ? sv.y : 0.f;
            } else {
                mx[e & 1] = max3(mx[e & 1], sv.x, sv.y);
                x = f2_fma(sv, sc2, nm);
            }
            a1 = f2_add(a1, sv);
            a2 = f2_fma(sv, sv, a2);
            float2 p;
            if (!kDiag && kPoly && ((POLAR_TC_POLY_MASK >> e) & 1)) {
                p = exp2_poly2(make_float2(fmaxf(x.x, -126.f), fmaxf(x.y, -126.f)));
            } else {
                p.x = ex2(x.x);
                p.y = ex2(x.y);
            }
            la = f2_add(la, p);
            l2a = f2_fma(p, p, l2a);
            pk[cc][e] = pack_bf16(p.x, p.y);
        }
    }
    tmax = fmaxf(mx[0], mx[1]);
    ts1 = a1.x + a1.y;
    ts2 = a2.x + a2.y;
    tl = la.x + la.y;
    tl2 = l2a.x + l2a.y;
}

// Max of the visible raw dots of a half row (keys tlo .. thi of the half when
// kDiag), and -- when it exceeds `above` -- the first visible key holding it
// (in *arg; otherwise *arg is left alone).  The backward's rows pass calls this
// before fused_half<.., kMax = false>, so the search runs while the raw dots
// are the only tile data in registers.
template <bool kDiag>
__device__ __forceinline__ float tile_max_half(const uint32_t (&sr)[2][32], int thi, int tlo,
                                               float above, int *arg) {
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int e = 0; e < 64; e += 2) {
        const float x0 = __uint_as_float(sr[e >> 5][e & 31]), x1 = __uint_as_float(sr[e >> 5][(e & 31) + 1]);
        if (kDiag)
            mx[(e >> 1) & 1] = max3(mx[(e >> 1) & 1], (e <= thi && e >= tlo) ? x0 : -INFINITY,
                                    (e + 1 <= thi && e + 1 >= tlo) ? x1 : -INFINITY);
        else
            mx[(e >> 1) & 1] = max3(mx[(e >> 1) & 1], x0, x1);
    }
    const float tmax = fmaxf(mx[0], mx[1]);
    if (tmax > above) {
        int idx = 64;
#pragma unroll
        for (int e = 63; e >= 0; --e) {
            const bool hit = __uint_as_float(sr[e >> 5][e & 31]) == tmax;
            idx = (kDiag ? hit && e <= thi && e >= tlo : hit) ? e : idx;
        }
        *arg = idx;
    }
    return tmax;
}

// fused_tile for a half row: 64 keys (keys 64*half .. 64*half + 63 of the
// tile, in sr[0..1][0..31]) of one row, used when two softmax threads share a
// row.  Key c of this half is visible iff tlo <= c <= thi (both in the half's
// own coordinates).
template <bool kDiag, bool kMoments, bool kMax = true>
__device__ __forceinline__ void fused_half(const uint32_t (&sr)[2][32], int thi, int tlo, float2 sc2,
                                           float neg_m, uint32_t (&pk)[2][16], float &tmax,
                                           float &ts1, float &ts2, float &tl, float &tl2) {
    const float2 nm = make_float2(neg_m, neg_m);
    float mx[2] = {-INFINITY, -INFINITY};
    float2 a1 = make_float2(0.f, 0.f), a2 = a1, la = a1, l2a = a1;
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) {
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            float2 sv = make_float2(__uint_as_float(sr[cc][2 * e]), __uint_as_float(sr[cc][2 * e + 1]));
            float2 x;
            if (kDiag) {
                const int col = 32 * cc + 2 * e;
                const bool v0 = col <= thi && col >= tlo, v1 = col + 1 <= thi && col + 1 >= tlo;
                if (kMax) mx[e & 1] = max3(mx[e & 1], v0 ? sv.x : -INFINITY, v1 ? sv.y : -INFINITY);
                x = f2_fma(sv, sc2, nm);
                x.x = v0 ? x.x : -INFINITY;
                x.y = v1 ? x.y : -INFINITY;
                sv.x = v0 ? sv.x : 0.f;
                sv.y = v1 ? sv.y : 0.f;
            } else {
                if (kMax) mx[e & 1] = max3(mx[e & 1], sv.x, sv.y);
                x = f2_fma(sv, sc2, nm);
            }
            if (kDiag || !kMoments) {  // full tiles: from the key moments instead
                a1 = f2_add(a1, sv);
                a2 = f2_fma(sv, sv, a2);
            }
            float2 p;
            if (!kDiag && ((POLAR_TC_SPLIT_POLY_MASK >> e) & 1)) {
                p = exp2_poly2(make_float2(fmaxf(x.x, -126.f), fmaxf(x.y, -126.f)));
            } else {
                p.x = ex2(x.x);
                p.y = ex2(x.y);
            }
            la = f2_add(la, p);
            l2a = f2_fma(p, p, l2a);
            pk[cc][e] = pack_bf16(p.x, p.y);
        }
    }
    tmax = fmaxf(mx[0], mx[1]);
    ts1 = a1.x + a1.y;
    ts2 = a2.x + a2.y;
    tl = la.x + la.y;
    tl2 = l2a.x + l2a.y;
}



struct TcArgs {
    const float *u;
    __nv_bfloat16 *out;
    float *neff;
    int *status;
    const float *mom;  // key-moment records (kMoments only)
    int B, T, Hq, Hkv, nqt, npairs;
    int window;  // 0: all causal keys; W > 0: the last W of each row's
    float s, alpha, L, beta, inv_ln_L;
    // Backward rows pass (kRows) only: the upstream gradient dL/dout
    // [B, T, Hq, 64] bf16, and the outputs the backward's tensor-core passes
    // read: per-row coefficient records [B][Hq][Tpad][kBwdCoefWords] and dA as
    // bf16 [B][Hq][Tpad][64] (Tpad = T rounded up to the 128-row tile).
    const __nv_bfloat16 *gout;
    float *coef;
    __nv_bfloat16 *dab;
    int Tpad;
    // The prefill's first query tile (a launch takes gridDim.x / (npairs B)
    // tiles from there).  Kept in the slot beside Tpad, so that the argument
    // block keeps its size (a larger one cost the training variant spills).
    int qt_lo;
    // Training forward (kSave) only: the saved row state [B][Hq][T][kFwdStateWords].
    float *state;
};

// Epilogue of one row: content = O/|O|, the magnitude channel from the row's
// streaming state, out = content + count (bf16, 128-bit stores) and n_eff.
// Returns |O| (floored at 1e-30).
__device__ __forceinline__ float store_row(const uint32_t (&o)[2][32], float l, float l2,
                                          float m_raw, float s1, float s2, float c, float n,
                                          const TcArgs &a, int b, int row, int h) {
    float ne;
    const float mag = polar_magnitude(l, l2, m_raw, s1, s2, c, n, a.beta, a.inv_ln_L, &ne);
    float nrm = 0.f;
#pragma unroll
    for (int hh = 0; hh < 2; ++hh)
#pragma unroll
        for (int e = 0; e < 32; ++e) {
            const float x = __uint_as_float(o[hh][e]);
            nrm = fmaf(x, x, nrm);
        }
    const float an = fmaxf(sqrtf(nrm), 1e-30f), inv = 1.0f / an;
    const float4 *u4 = reinterpret_cast<const float4 *>(a.u + static_cast<size_t>(h) * kHeadDim);
    uint4 *dst = reinterpret_cast<uint4 *>(a.out + ((static_cast<size_t>(b) * a.T + row) * a.Hq + h) *
                                                       kHeadDim);
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) {
        const float4 ua = __ldg(u4 + 2 * ch), ub = __ldg(u4 + 2 * ch + 1);
        const float uu[8] = {ua.x, ua.y, ua.z, ua.w, ub.x, ub.y, ub.z, ub.w};
        uint32_t w4[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int d0 = 8 * ch + 2 * e;
            const float x0 = __uint_as_float(o[d0 >> 5][d0 & 31]) * inv;
            const float x1 = __uint_as_float(o[(d0 + 1) >> 5][(d0 + 1) & 31]) * inv;
            w4[e] = pack_bf16(fmaf(mag, uu[2 * e], x0), fmaf(mag, uu[2 * e + 1], x1));
        }
        dst[ch] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
    }
    if (a.neff) a.neff[(static_cast<size_t>(b) * a.Hq + h) * a.T + row] = ne;
    return an;
}

// Epilogue of one row of the backward's rows pass (kRows): with content =
// O/|O| and g = dL/dout of the row, the chain rule through the magnitude
// channel (gate, tanh-log of n_eff, null floor) and the direction gives the
// row's coefficient record (BwdCoef layout, weights relative to the fixed
// reference cl2) and dA = (g - content <content, g>)/|O|, stored as bf16.  Rows
// past the end get zero dA and a record whose weights and dS vanish.  All 32
// lanes of the warp call this (tensor-memory loads are warp-collective).
__device__ __forceinline__ void store_rec(uint32_t tO, float l, float l2, float m_raw, int jarg,
                                          float s1, float s2, float c, float cl2, float n, int lo,
                                          const TcArgs &a, int b, int row, int h) {
    const bool live = row < a.T;
    const size_t rrow = (static_cast<size_t>(b) * a.Hq + h) * a.Tpad + row;
    const uint4 *gp = reinterpret_cast<const uint4 *>(
        a.gout + ((static_cast<size_t>(b) * a.T + (live ? row : 0)) * a.Hq + h) * kHeadDim);
    const float4 *u4 = reinterpret_cast<const float4 *>(a.u + static_cast<size_t>(h) * kHeadDim);
    // Pass 1, 16 dims at a time: |O|^2, <O, g>, <g, u_h>.
    float nrm = 0.f, og = 0.f, gu = 0.f;
#pragma unroll
    for (int ch = 0; ch < 4; ++ch) {
        uint32_t o[16];
        tmem_ld16(tO + 16 * ch, o);
        tmem_wait_ld();
        const uint4 g0 = live ? __ldg(gp + 2 * ch) : make_uint4(0u, 0u, 0u, 0u);
        const uint4 g1 = live ? __ldg(gp + 2 * ch + 1) : make_uint4(0u, 0u, 0u, 0u);
        const uint32_t gw[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float4 uu = __ldg(u4 + 4 * ch + q);
            const float ua[4] = {uu.x, uu.y, uu.z, uu.w};
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                const int e = 4 * q + x;
                const float gv = __uint_as_float(e & 1 ? gw[e >> 1] & 0xFFFF0000u : gw[e >> 1] << 16);
                const float ov = __uint_as_float(o[e]);
                nrm = fmaf(ov, ov, nrm);
                og = fmaf(ov, gv, og);
                gu = fmaf(gv, ua[x], gu);
            }
        }
    }
    const float nf = live ? n : 1.0f;
    const RowMag m = row_mag(l, l2, m_raw, s1, s2, c, nf, a.beta, a.inv_ln_L);
    const float an = fmaxf(sqrtf(nrm), 1e-30f), inv_an = 1.0f / an;
    const float cg = og * inv_an;  // <content, g>
    // Pass 2: dA = (g - O cg / |O|) / |O|.
    uint4 *dst = reinterpret_cast<uint4 *>(a.dab + rrow * kHeadDim);
    const float sc = inv_an * cg;
#pragma unroll
    for (int ch = 0; ch < 4; ++ch) {
        uint32_t o[16];
        tmem_ld16(tO + 16 * ch, o);
        tmem_wait_ld();
        const uint4 g0 = live ? __ldg(gp + 2 * ch) : make_uint4(0u, 0u, 0u, 0u);
        const uint4 g1 = live ? __ldg(gp + 2 * ch + 1) : make_uint4(0u, 0u, 0u, 0u);
        const uint32_t gw[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
        uint32_t d[8];
#pragma unroll
        for (int x = 0; x < 8; ++x) {
            const float g_lo = __uint_as_float(gw[x] << 16), g_hi = __uint_as_float(gw[x] & 0xFFFF0000u);
            const float d_lo = (g_lo - __uint_as_float(o[2 * x]) * sc) * inv_an;
            const float d_hi = (g_hi - __uint_as_float(o[2 * x + 1]) * sc) * inv_an;
            d[x] = live ? pack_bf16(d_lo, d_hi) : 0u;
        }
        dst[2 * ch] = make_uint4(d[0], d[1], d[2], d[3]);
        dst[2 * ch + 1] = make_uint4(d[4], d[5], d[6], d[7]);
    }
    store_coef_record(a.coef + rrow * kBwdCoefWords, live, m, gu, l, l2, c, cl2, nf, a.beta,
                      a.inv_ln_L, jarg, lo);
}

// kFixedRef: the exponentials use the fixed per-row reference m_ref = c*log2e,
// the largest logit L2-normalised q and k allow (|<q,k>| <= 1); weights then
// stay <= ~1 and no rescale is needed, so a tile's weights do not wait for
// its max.  A logit above the reference by more than the rescale threshold can
// only come from inputs that break the normalisation precondition; it is
// reported as POLAR_ERR_INVALID_ARG through the status word.
// The host picks kFixedRef only when the smallest weight squared, 2^(-4c*log2e),
// stays a normal fp32; otherwise the reference follows the running max.
// kSplit: softmax warpgroups per head slot.  1: one thread per row (128
// columns; any reference).  2: two threads per row, each with 64 of the keys
// (fixed reference only: the halves need no exchange until the epilogue).
// kMoments (split rows only): the raw sums S1, S2 of the null floor over the
// full key tiles come from the key moments of those tiles (sum k, sum k k^T;
// written by the moments pre-pass) instead of from every score: warp 3 adds the
// moment records up into shared memory during the main loop, and after the last
// score tile the score issuer computes Y_i = Q_i G on the tensor cores into the
// free score columns, so that S2_i = <Y_i, q_i> and S1_i = <sum k, q_i>.  The
// diagonal tile still sums its visible scores one by one.  The host uses this
// variant from kMomMinTiles query tiles on.
// kWindow: a sliding window shorter than the sequence (a.window); false
// compiles every window test away.
// kRows: the backward's rows pass -- the same forward sweep, which also finds
// each row's first argmax key, and the store_rec epilogue in place of the
// output (split rows, fixed reference, no key moments).
// kSave: the training forward -- the rows pass's sweep (with the argmax) and
// the forward's output, plus each row's streaming state (FwdState layout) for
// the backward.
template <bool kFixedRef, int kSplit, bool kMoments, bool kWindow, bool kRows = false,
          bool kSave = false>
__global__ void __launch_bounds__(128 + 256 * kSplit, 1)
fwd_tc_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
              const __grid_constant__ CUtensorMap tv, const TcArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = smem;                           // 2 tiles
    uint8_t *sK = smem + 2 * kTileBytes;          // kStagesKV tiles
    uint8_t *sV = sK + kStagesKV * kTileBytes;    // kStagesKV tiles
    uint8_t *sG = sV + kStagesKV * kTileBytes;    // key Gram, bf16 high part then low part
    float *sKs = reinterpret_cast<float *>(sG + 2 * kGramBytes);  // key sums, 64 fp32

    __shared__ __align__(8) uint64_t q_full, kv_full[kStagesKV], kv_empty[kStagesKV];
    __shared__ __align__(8) uint64_t s_full[2], s_free[2], p_full[2], pv_done[2], mma_done[2];
    __shared__ __align__(8) uint64_t g_full, y_full[2];
    __shared__ uint32_t tmem_base_sh;
    // kSplit == 2: per-row partial statistics of the upper key half
    // (m_raw, S1, S2, l, l2), handed to the lower half for the epilogue.
    __shared__ float part[kSplit == 2 ? 2 : 1][kSplit == 2 ? kBM : 1][6];
    static_assert(kSplit == 1 || kFixedRef, "split rows need the fixed reference");
    static_assert(!kMoments || kSplit == 2, "key moments are used by the split rows only");
    static_assert(!kRows || (kSplit == 2 && !kMoments), "the rows pass runs the split sweep");
    static_assert(!kSave || (kSplit == 2 && !kMoments && !kRows), "the training forward runs the split sweep");

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // Work tile: heaviest query tiles first (longest causal rows).
    const int per_qt = a.npairs * a.B;
    // (The backward's rows pass and the training forward always take every tile.)
    const int qt_top = kRows || kSave ? a.nqt : a.qt_lo + static_cast<int>(gridDim.x) / per_qt;
    const int qt = qt_top - 1 - static_cast<int>(blockIdx.x) / per_qt;
    const int rem = static_cast<int>(blockIdx.x) % per_qt;
    const int pair = rem % a.npairs, b = rem / a.npairs;
    const int h0 = 2 * pair;
    const int g = h0 / (a.Hq / a.Hkv);
    const int q0 = qt * kBM;
    // Key tiles jt0..qt are (partly) visible to some row of the tile; with a
    // sliding window the first is the one holding key q0 - window + 1.
    const int window = kWindow ? a.window : 0;
    const int jt0 = window > 0 ? max(0, q0 - window + 1) / kBN : 0;
    const int nkv = qt - jt0 + 1;
    // Loop tile j (key tile jt0 + j) needs masking if it is the diagonal tile
    // or starts before the window of the tile's last row (min(q0 + 127, T - 1)).
    auto masked_tile = [&](int j) {
        return j == nkv - 1 || (window > 0 && (jt0 + j) * kBN < min(q0 + kBM, a.T) - window);
    };
    // Key tiles every row of the tile sees in full: first_full() .. qt - 1 (the
    // unmasked loop tiles).  Their raw sums come from the key moments.
    auto first_full = [&]() {
        return window > 0 ? max(jt0, (min(q0 + kBM, a.T) - window + kBN - 1) / kBN) : 0;
    };
    // Visible key range of row t in loop tile j, in the tile's coordinates.
    auto vis_hi = [&](int j, int t) { return q0 + t - (jt0 + j) * kBN; };
    auto vis_lo = [&](int j, int t) {
        return window > 0 ? q0 + t - window + 1 - (jt0 + j) * kBN : -(1 << 30);
    };

    if (warp == 0 && lane == 0) {
        mbar_init(&q_full, 1);
        for (int st = 0; st < kStagesKV; ++st) {
            mbar_init(&kv_full[st], 1);
            mbar_init(&kv_empty[st], 2);  // one commit from each MMA issuer
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s_full[i], 1);
            mbar_init(&s_free[i], kBM * kSplit);
            mbar_init(&p_full[i], kBM * kSplit);
            mbar_init(&pv_done[i], 1);
        }
        mbar_init(&mma_done[0], 1);
        mbar_init(&mma_done[1], 1);
        mbar_init(&g_full, 1);
        mbar_init(&y_full[0], 1);
        mbar_init(&y_full[1], 1);
        fence_barrier_init();
    }
    if (warp == 1) tmem_alloc_512(&tmem_base_sh);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_sh;

    if (warp < 4) {
      reg_dealloc<64>();
      if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&tq);
            tma_prefetch_desc(&tk);
            tma_prefetch_desc(&tv);
            mbar_arrive_expect_tx(&q_full, 2 * kTileBytes);
            tma_load_4d(sQ, &tq, 0, h0, q0, b, &q_full);
            tma_load_4d(sQ + kTileBytes, &tq, 0, h0 + 1, q0, b, &q_full);
            int issued = 0;
            bool ok = true;
            for (int j = 0; j < nkv && ok; ++j) {
                const int st = j % kStagesKV;
                if (j >= kStagesKV) ok = mbar_wait(&kv_empty[st], ((j / kStagesKV) - 1) & 1, a.status);
                if (!ok) break;
                mbar_arrive_expect_tx(&kv_full[st], 2 * kTileBytes);
                tma_load_4d(sK + st * kTileBytes, &tk, 0, g, (jt0 + j) * kBN, b, &kv_full[st]);
                tma_load_4d(sV + st * kTileBytes, &tv, 0, g, (jt0 + j) * kBN, b, &kv_full[st]);
                ++issued;
            }
            // Every copy this thread started lands before shared memory is released.
            mbar_wait(&q_full, 0, a.status);
            for (int j = (issued > kStagesKV ? issued - kStagesKV : 0); j < issued; ++j)
                mbar_wait(&kv_full[j % kStagesKV], (j / kStagesKV) & 1, a.status);
        }
    } else if (warp == 1 || warp == 2) {
        // ------------------------------------------ MMA issuers (one thread each)
        // Warp 1 issues the score MMAs S_i(j) as soon as the K tile of j has landed
        // and softmax i has copied S_i(j-1) out of tensor memory; warp 2 issues the
        // PV MMAs as soon as P_i(j) is in tensor memory.  Neither waits behind the
        // other's backlog.  Each commits only the barriers that track its own MMAs
        // (a commit covers the issuing thread's MMAs); a K/V stage is free after
        // one commit from each.
        if (lane == 0) {
            constexpr uint32_t idesc_qk = idesc_bf16(kBM, kBN, false);
            constexpr uint32_t idesc_pv = idesc_bf16(kBM, kHeadDim, true);
            const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK), sVa = smem_u32(sV);
            // Descriptor halves: low = (address >> 4) | (LBO >> 4) << 16, high =
            // (SBO >> 4) | version 1 << 14 | SWIZZLE_128B << 29.  Q and K are
            // K-major (LBO 16, SBO 1024); V is MN-major (LBO 8192, SBO 1024).
            const uint32_t hi = (1024u >> 4) | (1u << 14) | (2u << 29);
            const uint32_t q_lo0 = ((sQa & 0x3FFFFu) >> 4) | (1u << 16);
            const uint32_t k_lo0 = ((sKa & 0x3FFFFu) >> 4) | (1u << 16);
            const uint32_t v_lo0 = ((sVa & 0x3FFFFu) >> 4) | ((8192u >> 4) << 16);
            constexpr uint32_t kStage = kTileBytes >> 4;
            auto issue_s = [&](int i, int j) {
                const uint32_t qa = q_lo0 + i * kStage, ka = k_lo0 + (j % kStagesKV) * kStage;
                const uint32_t d = tmem + (i ? kColS1 : kColS0);
                mma_ss2<0>(d, qa, hi, ka, hi, idesc_qk);
                mma_ss2<1>(d, qa + 2, hi, ka + 2, hi, idesc_qk);
                mma_ss2<1>(d, qa + 4, hi, ka + 4, hi, idesc_qk);
                mma_ss2<1>(d, qa + 6, hi, ka + 6, hi, idesc_qk);
                tc_commit(&s_full[i]);
            };
            auto issue_pv = [&](int i, int j) {
                const uint32_t va = v_lo0 + (j % kStagesKV) * kStage;
                const uint32_t d = tmem + (i ? kColO1 : kColO0), pa = tmem + (i ? kColP1 : kColP0);
                const uint32_t acc0 = j > 0;
                mma_ts2(d, pa, va, hi, idesc_pv, acc0);
#pragma unroll
                for (int kk = 1; kk < kBN / 16; ++kk)
                    mma_ts2(d, pa + 8 * kk, va + 128 * kk, hi, idesc_pv, 1u);
            };
            bool ok = true;
            if (warp == 1) {
                ok = mbar_wait(&q_full, 0, a.status);
#pragma unroll 1
                for (int j = 0; j < nkv && ok; ++j) {
                    if (!(ok = mbar_wait(&kv_full[j % kStagesKV], (j / kStagesKV) & 1, a.status))) break;
#pragma unroll 1
                    for (int i = 0; i < 2 && ok; ++i) {
                        if (j > 0 && !(ok = mbar_wait(&s_free[i], (j - 1) & 1, a.status))) break;
                        tc_fence_after();
                        issue_s(i, j);
                    }
                    if (ok) tc_commit(&kv_empty[j % kStagesKV]);
                }
                if constexpr (kMoments) {
                    // Y_i = Q_i (G_hi + G_lo) into S_i's first 64 columns, once
                    // softmax i has copied out its last score tile.
                    if (ok && first_full() <= qt - 1) {
                        constexpr uint32_t idesc_y = idesc_bf16(kBM, kHeadDim, false);
                        const uint32_t gh = ((smem_u32(sG) & 0x3FFFFu) >> 4) | (1u << 16);
                        const uint32_t gl = gh + (kGramBytes >> 4);
                        ok = mbar_wait(&g_full, 0, a.status);
                        for (int i = 0; i < 2 && ok; ++i) {
                            if (!(ok = mbar_wait(&s_free[i], (nkv - 1) & 1, a.status))) break;
                            tc_fence_after();
                            const uint32_t qa = q_lo0 + i * kStage;
                            const uint32_t d = tmem + (i ? kColS1 : kColS0);
                            mma_ss2<0>(d, qa, hi, gh, hi, idesc_y);
#pragma unroll
                            for (int kk = 1; kk < 4; ++kk)
                                mma_ss2<1>(d, qa + 2 * kk, hi, gh + 2 * kk, hi, idesc_y);
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk)
                                mma_ss2<1>(d, qa + 2 * kk, hi, gl + 2 * kk, hi, idesc_y);
                            tc_commit(&y_full[i]);
                        }
                    }
                }
            } else {
                for (int j = 0; j < nkv && ok; ++j) {
                    if (!(ok = mbar_wait(&kv_full[j % kStagesKV], (j / kStagesKV) & 1, a.status))) break;
                    for (int i = 0; i < 2 && ok; ++i) {
                        if (!(ok = mbar_wait(&p_full[i], j & 1, a.status))) break;
                        tc_fence_after();
                        issue_pv(i, j);
                        tc_commit(&pv_done[i]);
                    }
                    if (ok) tc_commit(&kv_empty[j % kStagesKV]);
                }
            }
            // All MMAs this thread issued complete before tensor memory is freed.
            tc_commit(&mma_done[warp - 1]);
            mbar_wait(&mma_done[warp - 1], 0, a.status);
        }
      } else if constexpr (kMoments) {
        // ----------------------------------------- warp 3: key moments
        // Moments of keys 0 .. q0-1: the records closing every chunk before
        // tile qt-1's, plus tile qt-1's own record.  The Gram goes to shared
        // memory as an MMA B operand (K-major, 128B-swizzled, one row of 64
        // bf16 per d) split into a bf16 high part and the bf16 of the remainder,
        // so that Q G_hi + Q G_lo carries the Gram to ~2^-16 relative; the key
        // sums stay fp32.
        const int jfull = first_full();
        if (jfull <= qt - 1) {
            constexpr int kRec4 = kMomFloats / 4;
            const float4 *rec = reinterpret_cast<const float4 *>(a.mom) +
                                (static_cast<size_t>(b) * a.Hkv + g) * (a.nqt - 1) * kRec4;
            // Moments of key tiles 0 .. t: the records closing the chunks before
            // t's, plus t's own running record.
            auto prefix = [&](int t, int i) {
                float4 v = rec[static_cast<size_t>(t) * kRec4 + i];
#pragma unroll 4
                for (int c = 0; c < t / kMomChunk; ++c) {
                    const float4 w = rec[static_cast<size_t>((c + 1) * kMomChunk - 1) * kRec4 + i];
                    v.x += w.x; v.y += w.y; v.z += w.z; v.w += w.w;
                }
                return v;
            };
            // Moments of key tiles lo .. hi (lo > 0): the records closing the
            // whole chunks between, hi's running record, and lo's chunk from lo
            // on (its closing record minus the running record before lo).
            auto range = [&](int lo, int hi, int i) {
                const int clo = lo / kMomChunk, chi = hi / kMomChunk;
                float4 v = rec[static_cast<size_t>(hi) * kRec4 + i];
                if (clo < chi) {
                    const float4 w = rec[static_cast<size_t>(clo * kMomChunk + kMomChunk - 1) * kRec4 + i];
                    v.x += w.x; v.y += w.y; v.z += w.z; v.w += w.w;
                    for (int c = clo + 1; c < chi; ++c) {
                        const float4 u = rec[static_cast<size_t>(c * kMomChunk + kMomChunk - 1) * kRec4 + i];
                        v.x += u.x; v.y += u.y; v.z += u.z; v.w += u.w;
                    }
                }
                if (lo % kMomChunk != 0) {
                    const float4 u = rec[static_cast<size_t>(lo - 1) * kRec4 + i];
                    v.x -= u.x; v.y -= u.y; v.z -= u.z; v.w -= u.w;
                }
                return v;
            };
            for (int i = lane; i < kRec4; i += 32) {
                // Tiles jfull .. qt - 1 (under a window, a range of a few chunks).
                const float4 v = jfull > 0 ? range(jfull, qt - 1, i) : prefix(qt - 1, i);
                if (i < kHeadDim * kHeadDim / 4) {
                    const int d = i >> 4, e0 = (i & 15) * 4;
                    const uint32_t off = d * 128 + ((((e0 >> 3) ^ (d & 7))) << 4) + (e0 & 7) * 2;
                    const uint32_t h01 = pack_bf16(v.x, v.y), h23 = pack_bf16(v.z, v.w);
                    const uint32_t l01 = pack_bf16(v.x - __uint_as_float(h01 << 16),
                                                   v.y - __uint_as_float(h01 & 0xFFFF0000u));
                    const uint32_t l23 = pack_bf16(v.z - __uint_as_float(h23 << 16),
                                                   v.w - __uint_as_float(h23 & 0xFFFF0000u));
                    *reinterpret_cast<uint2 *>(sG + off) = make_uint2(h01, h23);
                    *reinterpret_cast<uint2 *>(sG + kGramBytes + off) = make_uint2(l01, l23);
                } else {
                    reinterpret_cast<float4 *>(sKs)[i - kHeadDim * kHeadDim / 4] = v;
                }
            }
            fence_proxy_async_smem();  // the tensor core reads sG through the async proxy
            __syncwarp();
            if (lane == 0) mbar_arrive(&g_full);
        }
      }
    } else if constexpr (kSplit == 2) {
        reg_alloc<104>();
        // --------------------------------- softmax: two warpgroups per head
        const int sw = warp - 4;                 // 0..15
        const int slot = sw >> 3;                // head slot
        const int half = (sw >> 2) & 1;          // keys 64*half .. 64*half + 63 of a tile
        const int wq = warp & 3;                 // TMEM lane quarter
        const int t = 32 * wq + lane;            // row within the tile = TMEM lane
        const int h = h0 + slot;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(32 * wq) << 16);
        const uint32_t tS = lane_base + (slot ? kColS1 : kColS0) + 64 * half;
        const uint32_t tP = lane_base + (slot ? kColP1 : kColP0) + 32 * half;
        const uint32_t tO = lane_base + (slot ? kColO1 : kColO0);
        const int row = q0 + t;
        // Visible keys of the row: row + 1, or the window.
        const float n = static_cast<float>(window > 0 ? min(row + 1, window) : row + 1);
        const float c = a.s * length_temperature(n, a.alpha, a.L);
        const float cl2 = c * kLog2e;
        const float m_ref = cl2;
        const float2 sc2 = make_float2(cl2, cl2);
        float m_raw = -INFINITY, l = 0.f, l2 = 0.f, s1 = 0.f, s2 = 0.f;
        int jarg = -1;  // kRows, kSave: the first key of the row's max raw dot
        bool ok = true;
        for (int j = 0; j < nkv; ++j) {
            ok = mbar_wait(&s_full[slot], j & 1, a.status);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            tc_fence_after();
            uint32_t sr[2][32];
            tmem_ld32(tS, sr[0]);
            tmem_ld32(tS + 32, sr[1]);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&s_free[slot]);
            uint32_t pk[2][16];
            float tmax, ts1, ts2, tl, tl2;
            if constexpr (kRows || kSave) {
                // A strictly larger tile max moves the argmax to this tile: its
                // first visible key holding that value (keys in ascending order).
                int idx = -1;
                if (masked_tile(j)) {
                    const int hi = vis_hi(j, t) - 64 * half, lo = vis_lo(j, t) - 64 * half;
                    tmax = tile_max_half<true>(sr, hi, lo, m_raw, &idx);
                    float unused;
                    fused_half<true, false, false>(sr, hi, lo, sc2, -m_ref, pk, unused, ts1, ts2, tl, tl2);
                } else {
                    tmax = tile_max_half<false>(sr, 0, 0, m_raw, &idx);
                    float unused;
                    fused_half<false, false, false>(sr, 0, 0, sc2, -m_ref, pk, unused, ts1, ts2, tl, tl2);
                }
                if (idx >= 0) jarg = (jt0 + j) * kBN + 64 * half + idx;
            } else {
                if (masked_tile(j))
                    fused_half<true, kMoments>(sr, vis_hi(j, t) - 64 * half, vis_lo(j, t) - 64 * half,
                                               sc2, -m_ref, pk, tmax, ts1, ts2, tl, tl2);
                else
                    fused_half<false, kMoments>(sr, 0, 0, sc2, -m_ref, pk, tmax, ts1, ts2, tl, tl2);
            }
            s1 += ts1;
            s2 += ts2;
            l += tl;
            l2 += tl2;
            m_raw = fmaxf(m_raw, tmax);
            if (tmax * cl2 > m_ref + kRescaleThreshold) record_error(a.status, POLAR_ERR_INVALID_ARG);
            if (j > 0) {
                ok = mbar_wait(&pv_done[slot], (j - 1) & 1, a.status);
                if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                tc_fence_after();
            }
            tmem_st16(tP, pk[0]);
            tmem_st16(tP + 16, pk[1]);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&p_full[slot]);
        }
        if constexpr (kMoments) {
            // Null-floor sums over the full tiles, from the key moments: this
            // thread's 32 of the 64 components of S1 = <sum k, q>, S2 = <G q, q>.
            if (ok && (kWindow ? first_full() <= qt - 1 : nkv > 1)) {
                // g_full orders warp 3's key-sum stores before the reads below.
                ok = mbar_wait(&y_full[slot], 0, a.status) && mbar_wait(&g_full, 0, a.status);
                if (__all_sync(0xffffffffu, ok)) {
                    tc_fence_after();
                    const uint8_t *qrow = sQ + slot * kTileBytes + t * 128;
                    float m1 = 0.f, m2 = 0.f;
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {  // 16 columns at a time
                        uint32_t y[16];
                        tmem_ld16(lane_base + (slot ? kColS1 : kColS0) + 32 * half + 16 * hh, y);
                        tmem_wait_ld();
                        const float *ks = sKs + 32 * half + 16 * hh;
#pragma unroll
                        for (int cc = 0; cc < 2; ++cc) {
                            const int ch = 4 * half + 2 * hh + cc;
                            const uint4 w =
                                *reinterpret_cast<const uint4 *>(qrow + ((ch ^ (t & 7)) << 4));
                            const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                            for (int x = 0; x < 4; ++x) {
                                const float qa = __uint_as_float(ww[x] << 16);
                                const float qb = __uint_as_float(ww[x] & 0xFFFF0000u);
                                const int e = 8 * cc + 2 * x;
                                m2 = fmaf(__uint_as_float(y[e]), qa, m2);
                                m2 = fmaf(__uint_as_float(y[e + 1]), qb, m2);
                                m1 = fmaf(ks[e], qa, m1);
                                m1 = fmaf(ks[e + 1], qb, m1);
                            }
                        }
                    }
                    s1 += m1;
                    s2 += m2;
                } else {
                    ok = false;
                }
            }
        }
        // Combine the two halves of every row; the lower half runs the epilogue.
        if (half == 1) {
            part[slot][t][0] = m_raw;
            part[slot][t][1] = s1;
            part[slot][t][2] = s2;
            part[slot][t][3] = l;
            part[slot][t][4] = l2;
            part[slot][t][5] = __int_as_float(jarg);
        }
        named_barrier(1 + slot, 256);
        if (half == 0) {
            if constexpr (kRows || kSave) {
                // The upper half's keys of a tile follow the lower half's, but tiles
                // interleave: on a tie the smaller key index is the first argmax.
                const float om = part[slot][t][0];
                const int oj = __float_as_int(part[slot][t][5]);
                if (om > m_raw || (om == m_raw && oj >= 0 && (jarg < 0 || oj < jarg))) jarg = oj;
            }
            m_raw = fmaxf(m_raw, part[slot][t][0]);
            s1 += part[slot][t][1];
            s2 += part[slot][t][2];
            l += part[slot][t][3];
            l2 += part[slot][t][4];
            if (ok) ok = mbar_wait(&pv_done[slot], (nkv - 1) & 1, a.status);
            if (__all_sync(0xffffffffu, ok)) {
                tc_fence_after();
                if constexpr (kRows) {
                    const int lo = window > 0 ? max(0, row - window + 1) : 0;
                    store_rec(tO, l, l2, m_raw, jarg, s1, s2, c, cl2, n, lo, a, b, row, h);
                } else {
                    uint32_t o[2][32];
                    tmem_ld32(tO, o[0]);
                    tmem_ld32(tO + 32, o[1]);
                    tmem_wait_ld();
                    if (row < a.T) {
                        const float an = store_row(o, l, l2, m_raw, s1, s2, c, n, a, b, row, h);
                        if constexpr (kSave) {
                            float4 *st = reinterpret_cast<float4 *>(
                                a.state + ((static_cast<size_t>(b) * a.Hq + h) * a.T + row) * kFwdStateWords);
                            st[0] = make_float4(l, l2, m_raw, s1);
                            st[1] = make_float4(s2, an, __int_as_float(jarg), 0.f);
                        }
                    }
                }
            }
        }
    } else {
        reg_alloc<216>();
        // ------------------------------------------------ softmax warpgroups
        const int slot = (warp - 4) >> 2;          // head slot 0 or 1
        const int t = threadIdx.x - 128 * (1 + slot);  // row within the tile = TMEM lane
        const int h = h0 + slot;
        const int wq = warp & 3;                   // this warp's TMEM lane quarter
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(32 * wq) << 16);
        const uint32_t tS = lane_base + (slot ? kColS1 : kColS0);
        const uint32_t tP = lane_base + (slot ? kColP1 : kColP0);
        const uint32_t tO = lane_base + (slot ? kColO1 : kColO0);
        const int row = q0 + t;
        // Visible keys of the row: row + 1, or the window.
        const float n = static_cast<float>(window > 0 ? min(row + 1, window) : row + 1);
        const float c = a.s * length_temperature(n, a.alpha, a.L);
        const float cl2 = c * kLog2e;

        // Running reference: a finite floor rather than -inf, so that a tile with
        // no visible key (a sliding window can start past the first loaded
        // tile) gives weights 2^(-inf) = 0 instead of -inf + inf; the first real
        // max still rescales by 2^(floor - max) = 0.
        float m_ref = kFixedRef ? cl2 : -1e30f;
        float m_raw = -INFINITY, l = 0.f, l2 = 0.f, s1 = 0.f, s2 = 0.f;
        const float2 sc2 = make_float2(cl2, cl2);
        // O_i *= r for this thread's row (a warp-collective TMEM round trip).
        auto rescale_o = [&](float r) {
            uint32_t o[2][32];
            tmem_ld32(tO, o[0]);
            tmem_ld32(tO + 32, o[1]);
            tmem_wait_ld();
#pragma unroll
            for (int hh = 0; hh < 2; ++hh)
#pragma unroll
                for (int e = 0; e < 32; ++e)
                    o[hh][e] = __float_as_uint(__uint_as_float(o[hh][e]) * r);
            tmem_st32(tO, o[0]);
            tmem_st32(tO + 32, o[1]);
        };
        bool ok = true;
        for (int j = 0; j < nkv; ++j) {
            ok = mbar_wait(&s_full[slot], j & 1, a.status);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            tc_fence_after();
            uint32_t sr[4][32];
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) tmem_ld32(tS + 32 * cc, sr[cc]);
            tmem_wait_ld();
            // S_i(j) is in registers: the MMA thread may overwrite it with S_i(j+1).
            tc_fence_before();
            mbar_arrive(&s_free[slot]);
            const bool diag = masked_tile(j);
            const int thi = vis_hi(j, t), tlo = vis_lo(j, t);
            uint32_t pk[4][16];
            float r = 1.f;
            bool need = false;
            if (kFixedRef) {
                float tmax, ts1, ts2, tl, tl2;
                if (diag)
                    fused_tile<true, false>(sr, thi, tlo, sc2, -m_ref, pk, tmax, ts1, ts2, tl, tl2);
                else
                    fused_tile<false, true>(sr, thi, tlo, sc2, -m_ref, pk, tmax, ts1, ts2, tl, tl2);
                s1 += ts1;
                s2 += ts2;
                l += tl;
                l2 += tl2;
                m_raw = fmaxf(m_raw, tmax);
                // A logit this far above the unit-vector bound means q or k was not
                // L2-normalised: the precondition is broken and is reported.
                if (tmax * cl2 > m_ref + kRescaleThreshold) record_error(a.status, POLAR_ERR_INVALID_ARG);
            } else {
                float tmax, ts1, ts2;
                if (diag)
                    row_stats<true>(sr, thi, tlo, tmax, ts1, ts2);
                else
                    row_stats<false>(sr, thi, tlo, tmax, ts1, ts2);
                s1 += ts1;
                s2 += ts2;
                m_raw = fmaxf(m_raw, tmax);
                const float zmax = tmax * cl2;
                need = zmax > m_ref + kRescaleThreshold;
                if (need) {
                    r = ex2(m_ref - zmax);  // 0 on the first tile
                    l *= r;
                    l2 *= r * r;
                    m_ref = zmax;
                }
                float tl, tl2;
                if (diag)
                    row_weights<false>(sr, sc2, -m_ref, pk, tl, tl2);
                else
                    row_weights<true>(sr, sc2, -m_ref, pk, tl, tl2);
                l += tl;
                l2 += tl2;
            }
            // PV_i(j-1) done: P_i may be overwritten and O_i is current.  Waiting only
            // now lets this tile's weights overlap PV_i(j-1).
            if (j > 0) {
                ok = mbar_wait(&pv_done[slot], (j - 1) & 1, a.status);
                if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                tc_fence_after();
            }
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) tmem_st16(tP + 16 * cc, pk[cc]);
            // Rescale the output accumulator when this row's reference max moved.
            if (!kFixedRef && j > 0 && __any_sync(0xffffffffu, need)) rescale_o(r);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&p_full[slot]);
        }
        if (ok) ok = mbar_wait(&pv_done[slot], (nkv - 1) & 1, a.status);
        if (__all_sync(0xffffffffu, ok)) {
            tc_fence_after();
            uint32_t o[2][32];
            tmem_ld32(tO, o[0]);
            tmem_ld32(tO + 32, o[1]);
            tmem_wait_ld();
            if (row < a.T) store_row(o, l, l2, m_raw, s1, s2, c, n, a, b, row, h);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc_512(tmem);
    }
}

__global__ void selftest_exp2_kernel(const float2 *x, float2 *poly, float2 *mufu, int npairs) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= npairs) return;
    const float2 v = x[i];
    poly[i] = exp2_poly2(v);
    mufu[i] = make_float2(ex2(v.x), ex2(v.y));
}

// Tensor maps of q [B, T, Hq, 64] and k, v [B, T, Hkv, 64] bf16 as 4-D tensors
// (d, head, t, b): tiles of 128 rows x 64 with the 128-byte swizzle.
bool make_qkv_maps(const void *q, const void *k, const void *v, int B, int T, int Hq, int Hkv,
                   CUtensorMap *tq, CUtensorMap *tk, CUtensorMap *tv) {
    const uint32_t box[4] = {kHeadDim, 1, 128, 1};
    const uint64_t qdims[4] = {kHeadDim, (uint64_t)Hq, (uint64_t)T, (uint64_t)B};
    const uint64_t qstr[3] = {kHeadDim * 2ull, (uint64_t)Hq * kHeadDim * 2, (uint64_t)T * Hq * kHeadDim * 2};
    const uint64_t kdims[4] = {kHeadDim, (uint64_t)Hkv, (uint64_t)T, (uint64_t)B};
    const uint64_t kstr[3] = {kHeadDim * 2ull, (uint64_t)Hkv * kHeadDim * 2,
                              (uint64_t)T * Hkv * kHeadDim * 2};
    return encode_tiled(tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(q), qdims, qstr, box,
                        CU_TENSOR_MAP_SWIZZLE_128B) == CUDA_SUCCESS &&
           encode_tiled(tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(k), kdims, kstr, box,
                        CU_TENSOR_MAP_SWIZZLE_128B) == CUDA_SUCCESS &&
           encode_tiled(tv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(v), kdims, kstr, box,
                        CU_TENSOR_MAP_SWIZZLE_128B) == CUDA_SUCCESS;
}

}  // namespace

bool fwd_tc_reads_moments(const FwdLaunch &a) {
    if (!a.moments || a.dtype != POLAR_BF16 || (a.Hq / a.Hkv) % 2 != 0) return false;
    const bool windowed = a.window > 0 && a.window < a.T;
    const int n_max = windowed ? a.window : a.T;
    const float cl2_max = a.s *
                          (n_max > a.L ? 1.0f + a.alpha * logf(static_cast<float>(n_max) / a.L) : 1.0f) *
                          1.4426950408889634f;
    if (cl2_max > 28.0f) return false;
    return windowed ? a.window >= kMomMinTiles * kBN : (a.T + kBM - 1) / kBM >= kMomMinTiles;
}

cudaError_t launch_fwd_tc(const FwdLaunch &a) {
    const int G = a.Hq / a.Hkv;
    if (a.dtype != POLAR_BF16 || G % 2 != 0) return cudaErrorNotSupported;
    static std::atomic<uint64_t> configured{0};
    static std::atomic<uint64_t> split_ok{0};  // per device: the split kernel's register plan holds
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = 1ull << (dev & 63);
    if (!(configured.load() & bit)) {
        const void *all[] = {reinterpret_cast<const void *>(fwd_tc_kernel<true, 2, true, false>),
                             reinterpret_cast<const void *>(fwd_tc_kernel<true, 2, false, false>),
                             reinterpret_cast<const void *>(fwd_tc_kernel<false, 1, false, false>),
                             reinterpret_cast<const void *>(fwd_tc_kernel<true, 2, false, true>),
                             reinterpret_cast<const void *>(fwd_tc_kernel<false, 1, false, true>),
                             reinterpret_cast<const void *>(fwd_tc_kernel<true, 2, true, true>)};
        for (const void *f : all) {
            e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
            if (e != cudaSuccess) return e;
        }
        // setmaxnreg can only hand out the registers the block was launched with:
        // 64 for the producer/MMA warpgroup plus 104 for each of the four softmax
        // warpgroups must fit in (registers per thread at launch) x 640.
        const long long need = 64ll * 128 + 104ll * 512;
        bool fits = true;
        for (int i = 0; i < 6; ++i) {
            if (i == 2 || i == 4) continue;  // the one-warpgroup-per-head kernels
            cudaFuncAttributes fa;
            e = cudaFuncGetAttributes(&fa, all[i]);
            if (e != cudaSuccess) return e;
            fits = fits && static_cast<long long>(fa.numRegs) * 640 >= need;
        }
        if (fits) split_ok.fetch_or(bit);
        configured.fetch_or(bit);
    }
    // [B, T, H, 64] bf16 as a 4-D tensor (d, head, t, b); tiles of 128 rows x 64.
    CUtensorMap tq, tk, tv;
    if (!make_qkv_maps(a.q, a.k, a.v, a.B, a.T, a.Hq, a.Hkv, &tq, &tk, &tv)) return cudaErrorInvalidValue;
    TcArgs ta = {};
    ta.u = a.u;
    ta.out = static_cast<__nv_bfloat16 *>(a.out);
    ta.neff = a.neff;
    ta.status = a.status;
    ta.mom = a.moments;
    ta.B = a.B; ta.T = a.T; ta.Hq = a.Hq; ta.Hkv = a.Hkv;
    ta.nqt = (a.T + kBM - 1) / kBM;
    if (a.qt_lo < 0 || a.qt_cnt < 0 || a.qt_lo + a.qt_cnt > ta.nqt) return cudaErrorInvalidValue;
    ta.qt_lo = a.qt_lo;
    const int qt_cnt = a.qt_cnt > 0 ? a.qt_cnt : ta.nqt - a.qt_lo;
    // A window no shorter than the sequence changes nothing.
    const bool windowed = a.window > 0 && a.window < a.T;
    ta.window = windowed ? a.window : 0;
    ta.npairs = a.Hq / 2;
    ta.s = a.s; ta.alpha = a.alpha; ta.L = static_cast<float>(a.L); ta.beta = a.beta;
    ta.inv_ln_L = 1.0f / logf(static_cast<float>(a.L));
    const long long ctas = static_cast<long long>(qt_cnt) * ta.npairs * a.B;
    if (ctas <= 0) return cudaSuccess;
    if (ctas > 0x7fffffffll) return cudaErrorInvalidValue;
    // Fixed exponential reference while the smallest weight squared, 2^(-4 c_max log2e)
    // with c_max the largest logit scale of any row, stays well inside fp32.
    const int n_max = windowed ? a.window : a.T;  // longest visible range
    const float cl2_max = a.s *
                          (n_max > a.L ? 1.0f + a.alpha * logf(static_cast<float>(n_max) / a.L) : 1.0f) *
                          1.4426950408889634f;
    const unsigned grid = static_cast<unsigned>(ctas);
    // The records the launch's query tiles read: those of key tiles below its
    // last query tile, from the chunk holding its first query tile's.
    const int rec_lo = ta.qt_lo > 0 ? ta.qt_lo - 1 : 0, rec_hi = ta.qt_lo + qt_cnt - 1;
    if (cl2_max <= 28.0f && (split_ok.load() & bit)) {
        if (windowed && a.moments && a.window >= kMomMinTiles * kBN) {
            // A window of at least kMomMinTiles tiles: the full tiles' raw sums
            // from differences of key-moment prefixes (every record below rec_hi).
            if (!a.moments_ready) {
                e = launch_fwd_moments(a.k, a.B, a.T, a.Hkv, a.moments, 0, rec_hi, a.stream);
                if (e != cudaSuccess) return e;
            }
            fwd_tc_kernel<true, 2, true, true><<<grid, 640, kSmemBytes, a.stream>>>(tq, tk, tv, ta);
        } else if (windowed) {
            fwd_tc_kernel<true, 2, false, true><<<grid, 640, kSmemBytes, a.stream>>>(tq, tk, tv, ta);
        } else if (a.moments && ta.nqt >= kMomMinTiles) {
            if (!a.moments_ready) {
                e = launch_fwd_moments(a.k, a.B, a.T, a.Hkv, a.moments, rec_lo, rec_hi, a.stream);
                if (e != cudaSuccess) return e;
            }
            fwd_tc_kernel<true, 2, true, false><<<grid, 640, kSmemBytes, a.stream>>>(tq, tk, tv, ta);
        } else {
            fwd_tc_kernel<true, 2, false, false><<<grid, 640, kSmemBytes, a.stream>>>(tq, tk, tv, ta);
        }
    } else if (windowed) {
        fwd_tc_kernel<false, 1, false, true><<<grid, 384, kSmemBytes, a.stream>>>(tq, tk, tv, ta);
    } else {
        fwd_tc_kernel<false, 1, false, false><<<grid, 384, kSmemBytes, a.stream>>>(tq, tk, tv, ta);
    }
    count_launches(1);
    return cudaGetLastError();
}

// The backward's rows pass on the tensor cores: the forward sweep of every
// (query tile, head pair) with the store_rec epilogue.  Returns
// cudaErrorNotSupported where this kernel does not apply (fp32 inputs, an odd
// group size, a logit scale past the fixed reference's range, or a device
// whose register plan does not hold); the caller then uses its own rows pass.
cudaError_t launch_bwd_rows_tc(const BwdLaunch &l, float *coef, void *dab, int Tpad) {
    const int G = l.Hq / l.Hkv;
    if (l.dtype != POLAR_BF16 || G % 2 != 0) return cudaErrorNotSupported;
    const bool windowed = l.window > 0 && l.window < l.T;
    const int n_max = windowed ? l.window : l.T;
    const float cl2_max = l.s * (n_max > l.L ? 1.0f + l.alpha * logf(static_cast<float>(n_max) / l.L)
                                             : 1.0f) * 1.4426950408889634f;
    if (cl2_max > 28.0f) return cudaErrorNotSupported;
    static std::atomic<uint64_t> configured{0};
    static std::atomic<uint64_t> plan_ok{0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = 1ull << (dev & 63);
    const void *fns[] = {reinterpret_cast<const void *>(fwd_tc_kernel<true, 2, false, false, true>),
                         reinterpret_cast<const void *>(fwd_tc_kernel<true, 2, false, true, true>)};
    if (!(configured.load() & bit)) {
        bool fits = true;
        for (const void *f : fns) {
            e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
            if (e != cudaSuccess) return e;
            cudaFuncAttributes fa;
            e = cudaFuncGetAttributes(&fa, f);
            if (e != cudaSuccess) return e;
            fits = fits && static_cast<long long>(fa.numRegs) * 640 >= 64ll * 128 + 104ll * 512;
        }
        if (fits) plan_ok.fetch_or(bit);
        configured.fetch_or(bit);
    }
    if (!(plan_ok.load() & bit)) return cudaErrorNotSupported;
    CUtensorMap tq, tk, tv;
    if (!make_qkv_maps(l.q, l.k, l.v, l.B, l.T, l.Hq, l.Hkv, &tq, &tk, &tv)) return cudaErrorInvalidValue;
    TcArgs ta = {};
    ta.u = l.u;
    ta.status = l.status;
    ta.B = l.B; ta.T = l.T; ta.Hq = l.Hq; ta.Hkv = l.Hkv;
    ta.nqt = Tpad / kBM;
    ta.qt_lo = 0;
    ta.npairs = l.Hq / 2;
    ta.window = windowed ? l.window : 0;
    ta.s = l.s; ta.alpha = l.alpha; ta.L = static_cast<float>(l.L); ta.beta = l.beta;
    ta.inv_ln_L = 1.0f / logf(static_cast<float>(l.L));
    ta.gout = static_cast<const __nv_bfloat16 *>(l.dout);
    ta.coef = coef;
    ta.dab = static_cast<__nv_bfloat16 *>(dab);
    ta.Tpad = Tpad;
    const long long ctas = static_cast<long long>(ta.nqt) * ta.npairs * l.B;
    if (ctas <= 0) return cudaSuccess;
    if (ctas > 0x7fffffffll) return cudaErrorInvalidValue;
    const unsigned grid = static_cast<unsigned>(ctas);
    if (windowed)
        fwd_tc_kernel<true, 2, false, true, true><<<grid, 640, kSmemBytes, l.stream>>>(tq, tk, tv, ta);
    else
        fwd_tc_kernel<true, 2, false, false, true><<<grid, 640, kSmemBytes, l.stream>>>(tq, tk, tv, ta);
    count_launches(1);
    return cudaGetLastError();
}

// Per device: the training forward's register plan holds (bit set) and has
// been checked (bit set in state_checked).
static std::atomic<uint64_t> state_checked{0};
static std::atomic<uint64_t> state_plan_ok{0};

static cudaError_t check_state_plan(int dev, bool *ok) {
    const uint64_t bit = 1ull << (dev & 63);
    if (!(state_checked.load() & bit)) {
        const void *fns[] = {
            reinterpret_cast<const void *>(fwd_tc_kernel<true, 2, false, false, false, true>),
            reinterpret_cast<const void *>(fwd_tc_kernel<true, 2, false, true, false, true>)};
        bool fits = true;
        for (const void *f : fns) {
            cudaError_t e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
            if (e != cudaSuccess) return e;
            cudaFuncAttributes fa;
            e = cudaFuncGetAttributes(&fa, f);
            if (e != cudaSuccess) return e;
            fits = fits && static_cast<long long>(fa.numRegs) * 640 >= 64ll * 128 + 104ll * 512;
        }
        if (fits) state_plan_ok.fetch_or(bit);
        state_checked.fetch_or(bit);
    }
    *ok = (state_plan_ok.load() & bit) != 0;
    return cudaSuccess;
}

int fwd_state_supported(int dtype, int T, int Hq, int Hkv, float s, float alpha, int L, int window) {
    if (dtype != POLAR_BF16 || Hkv <= 0 || (Hq / Hkv) % 2 != 0) return 0;
    const bool windowed = window > 0 && window < T;
    const int n_max = windowed ? window : T;
    const float cl2_max = s * (n_max > L ? 1.0f + alpha * logf(static_cast<float>(n_max) / L) : 1.0f) *
                          1.4426950408889634f;
    if (cl2_max > 28.0f) return 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    bool ok = false;
    if (check_state_plan(dev, &ok) != cudaSuccess) return -1;
    return ok ? 1 : 0;
}

// The training forward: the split kernel's sweep with the first-argmax search,
// the forward's output and n_eff, and each row's streaming state.
cudaError_t launch_fwd_train_tc(const FwdLaunch &a) {
    if (!a.state) return cudaErrorInvalidValue;
    const int sup = fwd_state_supported(a.dtype, a.T, a.Hq, a.Hkv, a.s, a.alpha, a.L, a.window);
    if (sup < 0) return cudaErrorUnknown;
    if (sup == 0) return cudaErrorNotSupported;
    CUtensorMap tq, tk, tv;
    if (!make_qkv_maps(a.q, a.k, a.v, a.B, a.T, a.Hq, a.Hkv, &tq, &tk, &tv)) return cudaErrorInvalidValue;
    TcArgs ta = {};
    ta.u = a.u;
    ta.out = static_cast<__nv_bfloat16 *>(a.out);
    ta.neff = a.neff;
    ta.status = a.status;
    ta.state = a.state;
    ta.B = a.B; ta.T = a.T; ta.Hq = a.Hq; ta.Hkv = a.Hkv;
    ta.nqt = (a.T + kBM - 1) / kBM;
    ta.qt_lo = 0;
    const bool windowed = a.window > 0 && a.window < a.T;
    ta.window = windowed ? a.window : 0;
    ta.npairs = a.Hq / 2;
    ta.s = a.s; ta.alpha = a.alpha; ta.L = static_cast<float>(a.L); ta.beta = a.beta;
    ta.inv_ln_L = 1.0f / logf(static_cast<float>(a.L));
    const long long ctas = static_cast<long long>(ta.nqt) * ta.npairs * a.B;
    if (ctas <= 0) return cudaSuccess;
    if (ctas > 0x7fffffffll) return cudaErrorInvalidValue;
    const unsigned grid = static_cast<unsigned>(ctas);
    if (windowed)
        fwd_tc_kernel<true, 2, false, true, false, true><<<grid, 640, kSmemBytes, a.stream>>>(tq, tk, tv, ta);
    else
        fwd_tc_kernel<true, 2, false, false, false, true><<<grid, 640, kSmemBytes, a.stream>>>(tq, tk, tv, ta);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace polar

extern "C" polar_status_t polar_attn_selftest_exp2(const float *x, float *poly, float *mufu, int n,
                                                   void *stream) {
    if (!x || !poly || !mufu || n < 0 || (n & 1)) return POLAR_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(poly) |
         reinterpret_cast<uintptr_t>(mufu)) & 7u)
        return POLAR_ERR_INVALID_ARG;
    if (n == 0) return POLAR_OK;
    const int np = n / 2;
    polar::selftest_exp2_kernel<<<(np + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(
        reinterpret_cast<const float2 *>(x), reinterpret_cast<float2 *>(poly),
        reinterpret_cast<float2 *>(mufu), np);
    polar::count_launches(1);
    return cudaGetLastError() == cudaSuccess ? POLAR_OK : POLAR_ERR_CUDA;
}
