// decode.cu -- GQA-grouped paged-KV Polar Attention decode for sm_100a.
//
// "GQA-Grouped Paged Decode Kernel" (ATMA technical summary, section 2.2):
// the query of each sequence is scored straight from the paged KV cache, and
// each key/value page is read from HBM once for all G = Hq/Hkv query heads of
// its group (a per-head kernel would read it G times).
//
// Two launches:
//  1. split kernel, grid (split, kv head, sequence): a CTA streams a run of
//     pages of one (sequence, kv head) through a TMA ring in shared memory and
//     keeps, per query head of the group, the streaming state of the method:
//     reference max, l = sum w, l2 = sum w^2 (rescaled by r and r^2 when the
//     max moves), the raw-dot sums for the null floor, and the value
//     accumulator.  It writes that state as a partial.
//  2. merge kernel, grid (query head, sequence): combines the partials exactly
//     (each rescaled to the common max: l by r, l2 by r^2, acc by r) and runs
//     the epilogue: content = acc/|acc|, n_eff = l^2/l2, null floor, gate,
//     count, out = content + count.
//
// The page pool is read through one 2D tensor map over rows of 64 bf16 (128
// bytes); each (page, K|V, head) block of 64 rows lands in shared memory with
// the 128-byte swizzle, so that the reads below are free of bank conflicts.
#include <algorithm>
#include <atomic>

#include "polar_common.cuh"
#include "polar_internal.h"

namespace polar {
namespace {

// Pages in flight per CTA.  Three stages (48 KB) let four CTAs share an SM;
// measured on B200 against 2, 4 and 6 stages, this is the fastest for one
// query token per sequence (0.964 ms, 4 stages 0.995) and for chunks of four
// (1.010 ms, 4 stages 1.169), which need more warps to hide their longer
// softmax per page.
constexpr int kStages = 3;
constexpr int kChunkBytes = kPage * kHeadDim * 2;      // one (page, K|V, head): 8 KB
constexpr int kStageBytes = 2 * kChunkBytes;           // K and V
constexpr int kPartialFloats = 72;                     // acc[64] + 6 stats + 2 pad
constexpr int kSplitSmem = kStages * kStageBytes + 1024;  // + alignment slack

struct SplitArgs {
    const int32_t *page_table;
    const int32_t *seqlens;
    const __nv_bfloat16 *q;
    float *partials;
    int *status;
    int num_pages, max_pages, Hq, Hkv, pages_per_split, max_splits;
    int chunk;  // query tokens per sequence (the last `chunk` cache positions)
    int window; // 0: every cached position; W > 0: each row's last W
    float s, alpha, L;
    int kv_div; // grid heads per kv head whose pages a CTA reads: 1, except in the
                // per-head self-test (one query head per CTA, so kv head = h / G)
};

// Page of the earliest cache position any query row of a sequence sees.
__host__ __device__ __forceinline__ int first_visible_page(int seqlen, int chunk, int window) {
    const int lo = window > 0 ? seqlen - chunk + 1 - window : 0;
    return lo > 0 ? lo / kPage : 0;
}

// Byte offset of logical 16-byte chunk c of row t inside a 128B-swizzled tile.
__device__ __forceinline__ uint32_t swz(int t, int c) {
    return static_cast<uint32_t>(t * 128 + ((c ^ (t & 7)) << 4));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

// d += A(16x16; a0/a2 row g of the lane, a1/a3 row g+8) * B(16x8), bf16 in,
// fp32 accumulate.
__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// Keep the low / high bf16 half of x only if the corresponding token is valid.
__device__ __forceinline__ uint32_t mask_pair(uint32_t x, bool lo_ok, bool hi_ok) {
    return (lo_ok ? (x & 0xFFFFu) : 0u) | (hi_ok ? (x & 0xFFFF0000u) : 0u);
}

// Split kernel: CTA (split, kv head g, sequence), 4 warps.  Warp w owns tokens
// 16w .. 16w+15 of every page.  The mma rows carry the R = G * chunk queries of
// the sequence that belong to kv head g: row r is query token r / G (of the
// chunk's `chunk` tokens, the last cache positions) for query head g*G + r % G;
// rows >= R are zero padding.  kTwo: R > 8, so rows 8-15 of the m16 tile carry
// queries too and each lane keeps two rows' state.  Each row keeps the
// streaming state of the method: reference max m_ref (log2 units), l, l2
// (rescaled by r, r^2 when m_ref moves past the lazy threshold), the raw-dot
// sums S1, S2 and max, and the value accumulator O (mma accumulator fragments).
// Row r sees the cache positions below n_r = seqlen - chunk + r / G + 1, so a
// chunk is causal within itself; its length temperature uses n_r.  The scores
// S = Q K^T and O += P V run on mma.sync (bf16 in, fp32 accumulate); the S
// fragments are reused as the P operand in registers.  At the end the four
// warps' states are merged exactly in shared memory into one partial per
// (split, row).
template <int G, bool kTwo>
__global__ void __launch_bounds__(128)
decode_split_kernel(const __grid_constant__ CUtensorMap kv_map, const SplitArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    constexpr int kHR = kTwo ? 2 : 1;       // row sets per lane: g and g + 8
    constexpr int kRows = 8 * kHR;
    __shared__ __align__(8) uint64_t full_bar[kStages];
    __shared__ float mst[4][kRows][6];          // per warp, row: m_ref, m_raw, l, l2, S1, S2
    // Per warp, row: the O row, in the page ring once every page is consumed
    // (so that four CTAs still fit per SM).
    static_assert(4 * kRows * kHeadDim * sizeof(float) <= kStages * kStageBytes, "ring too small");
    float(*macc)[kRows][kHeadDim] = reinterpret_cast<float(*)[kRows][kHeadDim]>(smem);

    const int split = blockIdx.x, g = blockIdx.y, seq = blockIdx.z;
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gq = lane >> 2, tq = lane & 3;  // mma row and column pair
    const int C = a.chunk, R = G * C;

    const int seqlen = a.seqlens[seq];
    if (seqlen < C || seqlen > a.max_pages * kPage) {
        if (split == 0 && g == 0 && threadIdx.x == 0) record_error(a.status, POLAR_ERR_BAD_SEQLEN);
        return;
    }
    const int npg = (seqlen + kPage - 1) / kPage;
    // Splits start at the page of the earliest position any row sees.
    const int p0 = first_visible_page(seqlen, C, a.window) + split * a.pages_per_split;
    if (p0 >= npg) return;
    const int np = min(npg, p0 + a.pages_per_split) - p0;
    const int32_t *pt = a.page_table + static_cast<size_t>(seq) * a.max_pages + p0;

    if (threadIdx.x == 0) {
        tma_prefetch_desc(&kv_map);
        for (int st = 0; st < kStages; ++st) mbar_init(&full_bar[st], 1);
        fence_barrier_init();
    }
    __syncthreads();

    // Producer: thread 0 fills a stage with the K and V blocks of one page.  A
    // page id outside the pool is reported and replaced by a plain arrive, so
    // the barrier phases stay in step.
    auto issue = [&](int kk) {
        const int st = kk % kStages;
        const int phys = pt[kk];
        if (phys >= 0 && phys < a.num_pages) {
            mbar_arrive_expect_tx(&full_bar[st], kStageBytes);
            const int row = (phys * 2 * a.Hkv + g / a.kv_div) * kPage;  // K block of the kv head
            tma_load_2d(smem + st * kStageBytes, &kv_map, 0, row, &full_bar[st]);
            tma_load_2d(smem + st * kStageBytes + kChunkBytes, &kv_map, 0, row + a.Hkv * kPage,
                        &full_bar[st]);
        } else {
            record_error(a.status, POLAR_ERR_BAD_PAGE);
            mbar_arrive(&full_bar[st]);
        }
    };
    if (threadIdx.x == 0)
        for (int kk = 0; kk < min(kStages, np); ++kk) issue(kk);

    // Per row set: query fragments (A operand of S = Q K^T), the visible
    // positions n_r and the row's exponent scale.
    uint32_t qa[kHR][4][2];
    int lim[kHR], lo[kHR];  // row r sees positions lo <= pos < lim
    float cl2[kHR];
#pragma unroll
    for (int hr = 0; hr < kHR; ++hr) {
        const int r = gq + 8 * hr;
        const bool real = r < R;
        const int t = real ? r / G : 0, hh = real ? r % G : 0;
        const uint32_t *qrow = reinterpret_cast<const uint32_t *>(
            a.q + ((static_cast<size_t>(seq) * C + t) * a.Hq + g * G + hh) * kHeadDim);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            qa[hr][kk][0] = real ? __ldg(qrow + 8 * kk + tq) : 0u;
            qa[hr][kk][1] = real ? __ldg(qrow + 8 * kk + 4 + tq) : 0u;
        }
        lim[hr] = seqlen - C + t + 1;
        lo[hr] = a.window > 0 ? max(0, lim[hr] - a.window) : 0;
        cl2[hr] = a.s * length_temperature(static_cast<float>(lim[hr] - lo[hr]), a.alpha, a.L) *
                  kLog2e;
    }

    float m_ref[kHR], m_raw[kHR], l[kHR], l2[kHR], s1[kHR], s2[kHR];
#pragma unroll
    for (int hr = 0; hr < kHR; ++hr) {
        m_ref[hr] = m_raw[hr] = -INFINITY;
        l[hr] = l2[hr] = s1[hr] = s2[hr] = 0.f;
    }
    float acc[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
    int issued = min(kStages, np), consumed = 0;
    bool ok = true;
    const uint32_t sbase = smem_u32(smem);

    for (int kk = 0; kk < np; ++kk) {
        const int st = kk % kStages;
        const uint32_t parity = (kk / kStages) & 1;
        const bool ready = mbar_wait(&full_bar[st], parity, a.status);
        if (!__syncthreads_and(ready)) { ok = false; break; }
        consumed = kk + 1;
        const int phys = pt[kk];
        if (phys >= 0 && phys < a.num_pages) {
            const int page = p0 + kk;
            const int ntok = page == npg - 1 ? seqlen - page * kPage : kPage;
            const uint32_t kb = sbase + st * kStageBytes, vb = kb + kChunkBytes;
            // S = Q K^T for this warp's 16 tokens (two n-tiles of 8).
            float sc[2][4];
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
                const int tok = 16 * w + 8 * nt + (lane & 7);
                uint32_t b[2][4];
                ldsm_x4(kb + swz(tok, lane >> 3), b[0]);
                ldsm_x4(kb + swz(tok, 4 + (lane >> 3)), b[1]);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(sc[nt], qa[0][ks][0], kTwo ? qa[kHR - 1][ks][0] : 0u, qa[0][ks][1],
                             kTwo ? qa[kHR - 1][ks][1] : 0u, b[ks >> 1][2 * (ks & 1)],
                             b[ks >> 1][2 * (ks & 1) + 1]);
            }
            // Streaming statistics of each row's visible positions (elements
            // 2hr, 2hr+1 of each n-tile belong to row set hr).
            uint32_t pa[kHR][2];
#pragma unroll
            for (int hr = 0; hr < kHR; ++hr) {
                const int pos0 = page * kPage + 16 * w + 2 * tq;
                bool vld[2][2];
                float tmax = -INFINITY, ts1 = 0.f, ts2 = 0.f;
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int pos = pos0 + 8 * nt + e;
                        vld[nt][e] = pos < lim[hr] && pos >= lo[hr];
                        const float x = sc[nt][2 * hr + e];
                        tmax = fmaxf(tmax, vld[nt][e] ? x : -INFINITY);
                        ts1 += vld[nt][e] ? x : 0.f;
                        ts2 += vld[nt][e] ? x * x : 0.f;
                    }
                tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 1));
                tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 2));
                s1[hr] += ts1;
                s2[hr] += ts2;
                m_raw[hr] = fmaxf(m_raw[hr], tmax);
                const float zmax = tmax * cl2[hr];
                if (zmax > m_ref[hr] + kRescaleThreshold) {  // uniform over the quad of the row
                    const float r = exp2f(m_ref[hr] - zmax);
                    l[hr] *= r;
                    l2[hr] *= r * r;
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        acc[i][2 * hr] *= r;
                        acc[i][2 * hr + 1] *= r;
                    }
                    m_ref[hr] = zmax;
                }
                float pv[2][2];
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const float pp =
                            vld[nt][e] ? exp2f(fmaf(sc[nt][2 * hr + e], cl2[hr], -m_ref[hr])) : 0.f;
                        pv[nt][e] = pp;
                        l[hr] += pp;
                        l2[hr] = fmaf(pp, pp, l2[hr]);
                    }
                pa[hr][0] = pack_bf16x2(pv[0][0], pv[0][1]);
                pa[hr][1] = pack_bf16x2(pv[1][0], pv[1][1]);
            }
            // O += P V: V^T fragments by transposed ldmatrix; tokens past the end
            // of the sequence are zeroed so no stale value can enter the sum.
            const bool last = ntok < kPage;
            const int trow = 16 * w + 8 * ((lane >> 3) & 1) + (lane & 7);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                uint32_t v[4];
                ldsm_x4_t(vb + swz(trow, 2 * i + (lane >> 4)), v);
                if (last) {
                    const int t0 = 16 * w + 2 * tq;
                    v[0] = mask_pair(v[0], t0 < ntok, t0 + 1 < ntok);
                    v[1] = mask_pair(v[1], t0 + 8 < ntok, t0 + 9 < ntok);
                    v[2] = mask_pair(v[2], t0 < ntok, t0 + 1 < ntok);
                    v[3] = mask_pair(v[3], t0 + 8 < ntok, t0 + 9 < ntok);
                }
                mma_bf16(acc[2 * i], pa[0][0], kTwo ? pa[kHR - 1][0] : 0u, pa[0][1],
                         kTwo ? pa[kHR - 1][1] : 0u, v[0], v[1]);
                mma_bf16(acc[2 * i + 1], pa[0][0], kTwo ? pa[kHR - 1][0] : 0u, pa[0][1],
                         kTwo ? pa[kHR - 1][1] : 0u, v[2], v[3]);
            }
        }
        __syncthreads();  // every warp is done with stage st
        if (threadIdx.x == 0 && issued < np) issue(issued++);
    }

    if (!ok) {
        // Bounded drain of copies still in flight before shared memory is released.
        if (threadIdx.x == 0)
            for (int kk = consumed; kk < issued; ++kk)
                mbar_wait(&full_bar[kk % kStages], (kk / kStages) & 1, a.status);
        __syncthreads();
        return;
    }

    // Reduce the quad of each row, then merge the four warps exactly.
#pragma unroll
    for (int hr = 0; hr < kHR; ++hr) {
#pragma unroll
        for (int o = 1; o <= 2; o <<= 1) {
            l[hr] += __shfl_xor_sync(0xffffffffu, l[hr], o);
            l2[hr] += __shfl_xor_sync(0xffffffffu, l2[hr], o);
            s1[hr] += __shfl_xor_sync(0xffffffffu, s1[hr], o);
            s2[hr] += __shfl_xor_sync(0xffffffffu, s2[hr], o);
            m_raw[hr] = fmaxf(m_raw[hr], __shfl_xor_sync(0xffffffffu, m_raw[hr], o));
        }
        const int r = gq + 8 * hr;
        if (r < R) {
            if (tq == 0) {
                mst[w][r][0] = m_ref[hr];
                mst[w][r][1] = m_raw[hr];
                mst[w][r][2] = l[hr];
                mst[w][r][3] = l2[hr];
                mst[w][r][4] = s1[hr];
                mst[w][r][5] = s2[hr];
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                macc[w][r][8 * i + 2 * tq] = acc[i][2 * hr];
                macc[w][r][8 * i + 2 * tq + 1] = acc[i][2 * hr + 1];
            }
        }
    }
    __syncthreads();
    for (int r = w; r < R; r += 4) {
        float M = -INFINITY;
#pragma unroll
        for (int ww = 0; ww < 4; ++ww) M = fmaxf(M, mst[ww][r][0]);
        float rr[4];
#pragma unroll
        for (int ww = 0; ww < 4; ++ww) rr[ww] = M == -INFINITY ? 0.f : exp2f(mst[ww][r][0] - M);
        float2 o = make_float2(0.f, 0.f);
        float ml = 0.f, ml2 = 0.f, ms1 = 0.f, ms2 = 0.f, mraw = -INFINITY;
#pragma unroll
        for (int ww = 0; ww < 4; ++ww) {
            o.x = fmaf(macc[ww][r][2 * lane], rr[ww], o.x);
            o.y = fmaf(macc[ww][r][2 * lane + 1], rr[ww], o.y);
            ml = fmaf(mst[ww][r][2], rr[ww], ml);
            ml2 = fmaf(mst[ww][r][3], rr[ww] * rr[ww], ml2);
            ms1 += mst[ww][r][4];
            ms2 += mst[ww][r][5];
            mraw = fmaxf(mraw, mst[ww][r][1]);
        }
        const int t = r / G, h = g * G + r % G;
        float *dst = a.partials +
                     (((static_cast<size_t>(seq) * C + t) * a.Hq + h) * a.max_splits + split) *
                         kPartialFloats;
        reinterpret_cast<float2 *>(dst)[lane] = o;
        if (lane == 0) {
            reinterpret_cast<float4 *>(dst + 64)[0] = make_float4(M, mraw, ml, ml2);
            reinterpret_cast<float2 *>(dst + 68)[0] = make_float2(ms1, ms2);
        }
    }
}

// Exact merge of the split partials of one (sequence, chunk token, query head)
// and the epilogue.  One warp; lane owns columns 2*lane and 2*lane + 1.
__global__ void __launch_bounds__(32)
decode_merge_kernel(const float *__restrict__ partials, const int32_t *__restrict__ seqlens,
                    const float *__restrict__ u, __nv_bfloat16 *__restrict__ out,
                    float *__restrict__ neff_out, int Hq, int chunk, int window, int max_pages,
                    int pages_per_split, int max_splits, float s, float alpha, float L, float beta,
                    float inv_ln_L) {
    const int h = blockIdx.x, row = blockIdx.y, lane = threadIdx.x;  // row = seq * chunk + token
    const int seq = row / chunk, tok = row % chunk;
    const int seqlen = seqlens[seq];
    if (seqlen < chunk || seqlen > max_pages * kPage) return;  // reported by the split kernel
    const int npg = (seqlen + kPage - 1) / kPage;
    const int nsplit =
        (npg - first_visible_page(seqlen, chunk, window) + pages_per_split - 1) / pages_per_split;
    const float *base = partials + (static_cast<size_t>(row) * Hq + h) * max_splits * kPartialFloats;

    float M = -INFINITY;
    for (int sp = lane; sp < nsplit; sp += 32) M = fmaxf(M, base[sp * kPartialFloats + 64]);
    M = warp_max(M);

    float l = 0.f, l2 = 0.f, s1 = 0.f, s2 = 0.f, m_raw = -INFINITY, a0 = 0.f, a1 = 0.f;
    for (int sp = 0; sp < nsplit; ++sp) {
        const float *p = base + sp * kPartialFloats;
        const float4 st = *reinterpret_cast<const float4 *>(p + 64);
        const float2 ss = *reinterpret_cast<const float2 *>(p + 68);
        const float2 ac = reinterpret_cast<const float2 *>(p)[lane];
        const float r = exp2f(st.x - M);  // st.x = the split's reference max (log2 units)
        l = fmaf(st.z, r, l);
        l2 = fmaf(st.w, r * r, l2);
        a0 = fmaf(ac.x, r, a0);
        a1 = fmaf(ac.y, r, a1);
        s1 += ss.x;
        s2 += ss.y;
        m_raw = fmaxf(m_raw, st.y);
    }
    const int lim = seqlen - chunk + tok + 1;  // positions below lim, the last `window` of them
    const float n = static_cast<float>(window > 0 ? min(lim, window) : lim);
    const float c = s * length_temperature(n, alpha, L);
    float ne;
    const float mag = polar_magnitude(l, l2, m_raw, s1, s2, c, n, beta, inv_ln_L, &ne);
    const float nrm = sqrtf(warp_sum(a0 * a0 + a1 * a1));
    const float inv = 1.0f / fmaxf(nrm, 1e-30f);
    const float2 uu = reinterpret_cast<const float2 *>(u + static_cast<size_t>(h) * kHeadDim)[lane];
    const __nv_bfloat162 o = __floats2bfloat162_rn(fmaf(mag, uu.x, a0 * inv), fmaf(mag, uu.y, a1 * inv));
    reinterpret_cast<__nv_bfloat162 *>(out + (static_cast<size_t>(row) * Hq + h) * kHeadDim)[lane] = o;
    if (neff_out && lane == 0) neff_out[static_cast<size_t>(row) * Hq + h] = ne;
}

template <int G, bool kTwo>
cudaError_t launch_split(const CUtensorMap &map, const SplitArgs &sa, int num_seqs,
                         cudaStream_t stream) {
    static std::atomic<uint64_t> configured{0};  // one bit per device
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = 1ull << (dev & 63);
    if (!(configured.load() & bit)) {
        e = cudaFuncSetAttribute(decode_split_kernel<G, kTwo>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, kSplitSmem);
        if (e != cudaSuccess) return e;
        configured.fetch_or(bit);
    }
    dim3 grid(sa.max_splits, sa.Hkv, num_seqs);
    decode_split_kernel<G, kTwo><<<grid, 128, kSplitSmem, stream>>>(map, sa);
    return cudaGetLastError();
}

template <int G>
cudaError_t launch_split_rows(const CUtensorMap &map, const SplitArgs &sa, int num_seqs,
                              cudaStream_t stream) {
    return G * sa.chunk > 8 ? launch_split<G, true>(map, sa, num_seqs, stream)
                            : launch_split<G, false>(map, sa, num_seqs, stream);
}

}  // namespace

int decode_pages_per_split(int num_seqs, int max_pages, int Hkv) {
    // Aim for several waves of CTAs over 148 SMs (3 resident per SM) while
    // keeping the partial states (about 1/60 of the KV bytes at 64 pages per
    // split) and the merge small.
    const long long work = static_cast<long long>(num_seqs) * Hkv * max_pages;
    int pps = 64;
    while (pps > 4 && work / pps < 148ll * 3 * 4) pps >>= 1;
    return pps;
}

size_t decode_partials_bytes(int num_seqs, int max_pages, int Hq, int Hkv, int chunk) {
    const int pps = decode_pages_per_split(num_seqs, max_pages, Hkv);
    const size_t max_splits = (static_cast<size_t>(max_pages) + pps - 1) / pps;
    return static_cast<size_t>(num_seqs) * chunk * Hq * max_splits * kPartialFloats * sizeof(float);
}

cudaError_t decode_preload() {
    // Querying a kernel's attributes loads its code onto the current device
    // (under lazy module loading that otherwise happens at its first launch).
    const void *all[] = {reinterpret_cast<const void *>(decode_split_kernel<1, false>),
                         reinterpret_cast<const void *>(decode_split_kernel<1, true>),
                         reinterpret_cast<const void *>(decode_split_kernel<2, false>),
                         reinterpret_cast<const void *>(decode_split_kernel<2, true>),
                         reinterpret_cast<const void *>(decode_split_kernel<4, false>),
                         reinterpret_cast<const void *>(decode_split_kernel<4, true>),
                         reinterpret_cast<const void *>(decode_split_kernel<8, false>),
                         reinterpret_cast<const void *>(decode_split_kernel<8, true>),
                         reinterpret_cast<const void *>(decode_merge_kernel)};
    for (const void *f : all) {
        cudaFuncAttributes fa;
        const cudaError_t e = cudaFuncGetAttributes(&fa, f);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

cudaError_t launch_decode(const DecodeLaunch &a) {
    const int G = a.per_head ? 1 : a.Hq / a.Hkv;
    const int pps = decode_pages_per_split(a.num_seqs, a.max_pages, a.Hkv);
    const int max_splits = (a.max_pages + pps - 1) / pps;

    CUtensorMap map;
    const uint64_t rows = static_cast<uint64_t>(a.num_pages) * 2 * a.Hkv * kPage;
    const uint64_t dims[2] = {static_cast<uint64_t>(kHeadDim), rows};
    const uint64_t strides[1] = {kHeadDim * 2};
    const uint32_t box[2] = {kHeadDim, kPage};
    if (encode_tiled(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(a.kv_pages), dims,
                     strides, box, CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;

    SplitArgs sa{a.page_table, a.seqlens, static_cast<const __nv_bfloat16 *>(a.q),
                 static_cast<float *>(a.workspace), a.status, a.num_pages, a.max_pages, a.Hq, a.Hkv,
                 pps, max_splits, a.chunk, a.window, a.s, a.alpha, static_cast<float>(a.L), 1};
    if (a.chunk < 1 || G * a.chunk > 16) return cudaErrorInvalidValue;
    if (a.per_head) {
        // Test-only: one query head per CTA (grid y over the query heads), each
        // reading its kv head's pages on its own, so that every page is read
        // once per query head instead of once per group.
        if (a.chunk != 1) return cudaErrorInvalidValue;
        sa.kv_div = a.Hq / a.Hkv;
        static std::atomic<uint64_t> configured{0};
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return e;
        const uint64_t bit = 1ull << (dev & 63);
        if (!(configured.load() & bit)) {
            e = cudaFuncSetAttribute(decode_split_kernel<1, false>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, kSplitSmem);
            if (e != cudaSuccess) return e;
            configured.fetch_or(bit);
        }
        decode_split_kernel<1, false><<<dim3(max_splits, a.Hq, a.num_seqs), 128, kSplitSmem,
                                        a.stream>>>(map, sa);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        dim3 mgrid(a.Hq, a.num_seqs);
        decode_merge_kernel<<<mgrid, 32, 0, a.stream>>>(
            static_cast<const float *>(a.workspace), a.seqlens, a.u,
            static_cast<__nv_bfloat16 *>(a.out), a.neff, a.Hq, 1, a.window, a.max_pages, pps,
            max_splits, a.s, a.alpha, static_cast<float>(a.L), a.beta,
            1.0f / logf(static_cast<float>(a.L)));
        count_launches(2);
        return cudaGetLastError();
    }
    cudaError_t e;
    switch (G) {
        case 1: e = launch_split_rows<1>(map, sa, a.num_seqs, a.stream); break;
        case 2: e = launch_split_rows<2>(map, sa, a.num_seqs, a.stream); break;
        case 4: e = launch_split_rows<4>(map, sa, a.num_seqs, a.stream); break;
        case 8: e = launch_split_rows<8>(map, sa, a.num_seqs, a.stream); break;
        default: return cudaErrorInvalidValue;
    }
    if (e != cudaSuccess) return e;
    dim3 mgrid(a.Hq, a.num_seqs * a.chunk);
    decode_merge_kernel<<<mgrid, 32, 0, a.stream>>>(
        static_cast<const float *>(a.workspace), a.seqlens, a.u, static_cast<__nv_bfloat16 *>(a.out),
        a.neff, a.Hq, a.chunk, a.window, a.max_pages, pps, max_splits, a.s, a.alpha,
        static_cast<float>(a.L), a.beta, 1.0f / logf(static_cast<float>(a.L)));
    count_launches(2);
    return cudaGetLastError();
}

}  // namespace polar
