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

constexpr int kStages = 4;                             // pages in flight per CTA
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
    float s, alpha, L;
};

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

// d += A(16x16, rows g and g+8 of the lane) * B(16x8), bf16 in, fp32 accumulate.
// Rows g+8 (a1, a3) are the zero padding of the query-head dimension.
__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a2, uint32_t b0,
                                         uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
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
// 16w .. 16w+15 of every page and keeps, for each query head of the group
// (mma rows; rows >= G are zero padding), the streaming state of the method:
// reference max m_ref (log2 units), l, l2 (rescaled by r, r^2 when m_ref
// moves past the lazy threshold), the raw-dot sums S1, S2 and max, and the
// value accumulator O (mma accumulator fragments).  The scores S = Q K^T and
// O += P V run on mma.sync (bf16 in, fp32 accumulate); the S fragments are
// reused as the P operand in registers.  At the end the four warps' states are
// merged exactly in shared memory into one partial per (split, query head).
template <int G>
__global__ void __launch_bounds__(128)
decode_split_kernel(const __grid_constant__ CUtensorMap kv_map, const SplitArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ __align__(8) uint64_t full_bar[kStages];
    __shared__ float mst[4][G][6];          // per warp, head: m_ref, m_raw, l, l2, S1, S2
    __shared__ float macc[4][G][kHeadDim];  // per warp, head: O row

    const int split = blockIdx.x, g = blockIdx.y, seq = blockIdx.z;
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gq = lane >> 2, tq = lane & 3;  // mma row (query head) and column pair

    const int seqlen = a.seqlens[seq];
    if (seqlen < 1 || seqlen > a.max_pages * kPage) {
        if (split == 0 && g == 0 && threadIdx.x == 0) record_error(a.status, POLAR_ERR_BAD_SEQLEN);
        return;
    }
    const int npg = (seqlen + kPage - 1) / kPage;
    const int p0 = split * a.pages_per_split;
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
            const int row = (phys * 2 * a.Hkv + g) * kPage;  // K block of head g
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

    // Query fragments (A operand of S = Q K^T): row gq = query head g*G + gq.
    const bool real = gq < G;
    uint32_t qa[4][2];
    {
        const uint32_t *qrow = reinterpret_cast<const uint32_t *>(
            a.q + (static_cast<size_t>(seq) * a.Hq + g * G + (real ? gq : 0)) * kHeadDim);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            qa[kk][0] = real ? __ldg(qrow + 8 * kk + tq) : 0u;
            qa[kk][1] = real ? __ldg(qrow + 8 * kk + 4 + tq) : 0u;
        }
    }
    const float n = static_cast<float>(seqlen);
    const float cl2 = a.s * length_temperature(n, a.alpha, a.L) * kLog2e;

    float m_ref = -INFINITY, m_raw = -INFINITY, l = 0.f, l2 = 0.f, s1 = 0.f, s2 = 0.f;
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
                    mma_bf16(sc[nt], qa[ks][0], qa[ks][1], b[ks >> 1][2 * (ks & 1)],
                             b[ks >> 1][2 * (ks & 1) + 1]);
            }
            // Streaming statistics of the valid tokens (rows gq; c0/c1 of each n-tile).
            bool vld[2][2];
            float tmax = -INFINITY, ts1 = 0.f, ts2 = 0.f;
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    vld[nt][e] = 16 * w + 8 * nt + 2 * tq + e < ntok;
                    const float x = sc[nt][e];
                    tmax = fmaxf(tmax, vld[nt][e] ? x : -INFINITY);
                    ts1 += vld[nt][e] ? x : 0.f;
                    ts2 += vld[nt][e] ? x * x : 0.f;
                }
            tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 1));
            tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 2));
            s1 += ts1;
            s2 += ts2;
            m_raw = fmaxf(m_raw, tmax);
            const float zmax = tmax * cl2;
            if (zmax > m_ref + kRescaleThreshold) {  // uniform over the quad of row gq
                const float r = exp2f(m_ref - zmax);
                l *= r;
                l2 *= r * r;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    acc[i][0] *= r;
                    acc[i][1] *= r;
                }
                m_ref = zmax;
            }
            float pv[2][2];
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const float pp = vld[nt][e] ? exp2f(fmaf(sc[nt][e], cl2, -m_ref)) : 0.f;
                    pv[nt][e] = pp;
                    l += pp;
                    l2 = fmaf(pp, pp, l2);
                }
            const uint32_t pa0 = pack_bf16x2(pv[0][0], pv[0][1]);
            const uint32_t pa2 = pack_bf16x2(pv[1][0], pv[1][1]);
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
                mma_bf16(acc[2 * i], pa0, pa2, v[0], v[1]);
                mma_bf16(acc[2 * i + 1], pa0, pa2, v[2], v[3]);
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
    for (int o = 1; o <= 2; o <<= 1) {
        l += __shfl_xor_sync(0xffffffffu, l, o);
        l2 += __shfl_xor_sync(0xffffffffu, l2, o);
        s1 += __shfl_xor_sync(0xffffffffu, s1, o);
        s2 += __shfl_xor_sync(0xffffffffu, s2, o);
        m_raw = fmaxf(m_raw, __shfl_xor_sync(0xffffffffu, m_raw, o));
    }
    if (real) {
        if (tq == 0) {
            mst[w][gq][0] = m_ref;
            mst[w][gq][1] = m_raw;
            mst[w][gq][2] = l;
            mst[w][gq][3] = l2;
            mst[w][gq][4] = s1;
            mst[w][gq][5] = s2;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            macc[w][gq][8 * i + 2 * tq] = acc[i][0];
            macc[w][gq][8 * i + 2 * tq + 1] = acc[i][1];
        }
    }
    __syncthreads();
    for (int hh = w; hh < G; hh += 4) {
        float M = -INFINITY;
#pragma unroll
        for (int ww = 0; ww < 4; ++ww) M = fmaxf(M, mst[ww][hh][0]);
        float r[4];
#pragma unroll
        for (int ww = 0; ww < 4; ++ww) r[ww] = M == -INFINITY ? 0.f : exp2f(mst[ww][hh][0] - M);
        float2 o = make_float2(0.f, 0.f);
        float ml = 0.f, ml2 = 0.f, ms1 = 0.f, ms2 = 0.f, mraw = -INFINITY;
#pragma unroll
        for (int ww = 0; ww < 4; ++ww) {
            o.x = fmaf(macc[ww][hh][2 * lane], r[ww], o.x);
            o.y = fmaf(macc[ww][hh][2 * lane + 1], r[ww], o.y);
            ml = fmaf(mst[ww][hh][2], r[ww], ml);
            ml2 = fmaf(mst[ww][hh][3], r[ww] * r[ww], ml2);
            ms1 += mst[ww][hh][4];
            ms2 += mst[ww][hh][5];
            mraw = fmaxf(mraw, mst[ww][hh][1]);
        }
        const int h = g * G + hh;
        float *dst = a.partials +
                     ((static_cast<size_t>(seq) * a.Hq + h) * a.max_splits + split) * kPartialFloats;
        reinterpret_cast<float2 *>(dst)[lane] = o;
        if (lane == 0) {
            reinterpret_cast<float4 *>(dst + 64)[0] = make_float4(M, mraw, ml, ml2);
            reinterpret_cast<float2 *>(dst + 68)[0] = make_float2(ms1, ms2);
        }
    }
}

// Exact merge of the split partials of one (sequence, query head) and the
// epilogue.  One warp; lane owns columns 2*lane and 2*lane + 1.
__global__ void __launch_bounds__(32)
decode_merge_kernel(const float *__restrict__ partials, const int32_t *__restrict__ seqlens,
                    const float *__restrict__ u, __nv_bfloat16 *__restrict__ out,
                    float *__restrict__ neff_out, int Hq, int max_pages, int pages_per_split,
                    int max_splits, float s, float alpha, float L, float beta, float inv_ln_L) {
    const int h = blockIdx.x, seq = blockIdx.y, lane = threadIdx.x;
    const int seqlen = seqlens[seq];
    if (seqlen < 1 || seqlen > max_pages * kPage) return;  // reported by the split kernel
    const int npg = (seqlen + kPage - 1) / kPage;
    const int nsplit = (npg + pages_per_split - 1) / pages_per_split;
    const float *base = partials + (static_cast<size_t>(seq) * Hq + h) * max_splits * kPartialFloats;

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
    const float n = static_cast<float>(seqlen);
    const float c = s * length_temperature(n, alpha, L);
    float ne;
    const float mag = polar_magnitude(l, l2, m_raw, s1, s2, c, n, beta, inv_ln_L, &ne);
    const float nrm = sqrtf(warp_sum(a0 * a0 + a1 * a1));
    const float inv = 1.0f / fmaxf(nrm, 1e-30f);
    const float2 uu = reinterpret_cast<const float2 *>(u + static_cast<size_t>(h) * kHeadDim)[lane];
    const __nv_bfloat162 o = __floats2bfloat162_rn(fmaf(mag, uu.x, a0 * inv), fmaf(mag, uu.y, a1 * inv));
    reinterpret_cast<__nv_bfloat162 *>(out + (static_cast<size_t>(seq) * Hq + h) * kHeadDim)[lane] = o;
    if (neff_out && lane == 0) neff_out[static_cast<size_t>(seq) * Hq + h] = ne;
}

template <int G>
cudaError_t launch_split(const CUtensorMap &map, const SplitArgs &sa, int num_seqs,
                         cudaStream_t stream) {
    static std::atomic<uint64_t> configured{0};  // one bit per device
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = 1ull << (dev & 63);
    if (!(configured.load() & bit)) {
        e = cudaFuncSetAttribute(decode_split_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kSplitSmem);
        if (e != cudaSuccess) return e;
        configured.fetch_or(bit);
    }
    dim3 grid(sa.max_splits, sa.Hkv, num_seqs);
    decode_split_kernel<G><<<grid, 128, kSplitSmem, stream>>>(map, sa);
    return cudaGetLastError();
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

size_t decode_partials_bytes(int num_seqs, int max_pages, int Hq, int Hkv) {
    const int pps = decode_pages_per_split(num_seqs, max_pages, Hkv);
    const size_t max_splits = (static_cast<size_t>(max_pages) + pps - 1) / pps;
    return static_cast<size_t>(num_seqs) * Hq * max_splits * kPartialFloats * sizeof(float);
}

cudaError_t launch_decode(const DecodeLaunch &a) {
    const int G = a.Hq / a.Hkv;
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
                 pps, max_splits, a.s, a.alpha, static_cast<float>(a.L)};
    cudaError_t e;
    switch (G) {
        case 1: e = launch_split<1>(map, sa, a.num_seqs, a.stream); break;
        case 2: e = launch_split<2>(map, sa, a.num_seqs, a.stream); break;
        case 4: e = launch_split<4>(map, sa, a.num_seqs, a.stream); break;
        case 8: e = launch_split<8>(map, sa, a.num_seqs, a.stream); break;
        default: return cudaErrorInvalidValue;
    }
    if (e != cudaSuccess) return e;
    dim3 mgrid(a.Hq, a.num_seqs);
    decode_merge_kernel<<<mgrid, 32, 0, a.stream>>>(
        static_cast<const float *>(a.workspace), a.seqlens, a.u, static_cast<__nv_bfloat16 *>(a.out),
        a.neff, a.Hq, a.max_pages, pps, max_splits, a.s, a.alpha, static_cast<float>(a.L), a.beta,
        1.0f / logf(static_cast<float>(a.L)));
    count_launches(2);
    return cudaGetLastError();
}

}  // namespace polar
