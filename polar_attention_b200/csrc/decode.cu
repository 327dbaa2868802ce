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
__device__ __forceinline__ int swz(int t, int c) { return t * 128 + ((c ^ (t & 7)) << 4); }

template <int G>
__global__ void __launch_bounds__(32 * G)
decode_split_kernel(const __grid_constant__ CUtensorMap kv_map, const SplitArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ __align__(8) uint64_t full_bar[kStages];
    __shared__ __align__(16) float ps[G][kPage];

    const int split = blockIdx.x, g = blockIdx.y, seq = blockIdx.z;
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = g * G + w;

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

    // The query row of head h, fp32, in every lane.
    float qr[kHeadDim];
    {
        const uint4 *qp = reinterpret_cast<const uint4 *>(
            a.q + (static_cast<size_t>(seq) * a.Hq + h) * kHeadDim);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const uint4 raw = __ldg(qp + c);
            const __nv_bfloat162 *pr = reinterpret_cast<const __nv_bfloat162 *>(&raw);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = __bfloat1622float2(pr[e]);
                qr[c * 8 + 2 * e] = f.x;
                qr[c * 8 + 2 * e + 1] = f.y;
            }
        }
    }
    const float n = static_cast<float>(seqlen);
    const float cl2 = a.s * length_temperature(n, a.alpha, a.L) * kLog2e;

    float m_ref = -INFINITY, m_raw = -INFINITY, l = 0.f, l2 = 0.f, s1 = 0.f, s2 = 0.f;
    float acc0 = 0.f, acc1 = 0.f;  // d = 2*lane, 2*lane + 1
    int issued = min(kStages, np), consumed = 0;
    bool ok = true;

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
            const uint8_t *kb = smem + st * kStageBytes;
            const uint8_t *vb = kb + kChunkBytes;
            // logits of tokens lane and lane + 32 for head h
            float sd[2];
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int t = lane + 32 * r;
                float acc = 0.f;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint4 raw = *reinterpret_cast<const uint4 *>(kb + swz(t, c));
                    const __nv_bfloat162 *pr = reinterpret_cast<const __nv_bfloat162 *>(&raw);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 f = __bfloat1622float2(pr[e]);
                        acc = fmaf(qr[c * 8 + 2 * e], f.x, acc);
                        acc = fmaf(qr[c * 8 + 2 * e + 1], f.y, acc);
                    }
                }
                sd[r] = acc;
            }
            const bool v0 = lane < ntok, v1 = lane + 32 < ntok;
            const float z0 = v0 ? sd[0] * cl2 : -INFINITY;
            const float z1 = v1 ? sd[1] * cl2 : -INFINITY;
            s1 += (v0 ? sd[0] : 0.f) + (v1 ? sd[1] : 0.f);
            s2 += (v0 ? sd[0] * sd[0] : 0.f) + (v1 ? sd[1] * sd[1] : 0.f);
            m_raw = fmaxf(m_raw, fmaxf(v0 ? sd[0] : -INFINITY, v1 ? sd[1] : -INFINITY));
            const float tmax = warp_max(fmaxf(z0, z1));
            if (tmax > m_ref + kRescaleThreshold) {  // warp-uniform
                const float r = exp2f(m_ref - tmax);
                l *= r;
                l2 *= r * r;
                acc0 *= r;
                acc1 *= r;
                m_ref = tmax;
            }
            const float pa = exp2f(z0 - m_ref), pb = exp2f(z1 - m_ref);
            l += pa + pb;
            l2 += pa * pa + pb * pb;
            ps[w][lane] = pa;
            ps[w][lane + 32] = pb;
            __syncwarp();
            // acc[d] += sum_t p_t v_t[d] for this lane's two columns
            const int cw = lane >> 2, sub = (lane & 3) * 4;
            for (int t = 0; t < ntok; ++t) {
                const float p = ps[w][t];
                const __nv_bfloat162 vv = *reinterpret_cast<const __nv_bfloat162 *>(
                    vb + t * 128 + ((cw ^ (t & 7)) << 4) + sub);
                const float2 f = __bfloat1622float2(vv);
                acc0 = fmaf(p, f.x, acc0);
                acc1 = fmaf(p, f.y, acc1);
            }
            __syncwarp();
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

    l = warp_sum(l);
    l2 = warp_sum(l2);
    s1 = warp_sum(s1);
    s2 = warp_sum(s2);
    m_raw = warp_max(m_raw);
    float *dst = a.partials +
                 ((static_cast<size_t>(seq) * a.Hq + h) * a.max_splits + split) * kPartialFloats;
    reinterpret_cast<float2 *>(dst)[lane] = make_float2(acc0, acc1);
    if (lane == 0) {
        reinterpret_cast<float4 *>(dst + 64)[0] = make_float4(m_ref, m_raw, l, l2);
        reinterpret_cast<float2 *>(dst + 68)[0] = make_float2(s1, s2);
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
    decode_split_kernel<G><<<grid, 32 * G, kSplitSmem, stream>>>(map, sa);
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
