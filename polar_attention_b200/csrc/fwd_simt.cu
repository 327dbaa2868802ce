// fwd_simt.cu -- CUDA-core (FFMA) causal Polar Attention prefill.
//
// The path for fp32 inputs, which must not be rounded to bf16 or tf32 on the
// way into a tensor core, and a cross-check for the tensor-core kernel on bf16
// inputs.  It streams the keys in tiles of 64 through shared memory and keeps
// the running max, l = sum w, l2 = sum w^2 and the value accumulator per query
// row ("Fused Polar Attention Kernel", section 2.2 of the ATMA technical
// summary: participation ratio online with streaming accumulators and squared
// correction factors).  One thread owns one query row; a block owns 128
// consecutive rows of one (batch, query head).
#include "polar_common.cuh"
#include "polar_internal.h"

namespace polar {
namespace {

constexpr int kRows = 128;   // query rows per block (one per thread)
constexpr int kKeyTile = 64; // keys staged in shared memory per step

template <typename T>
__global__ void __launch_bounds__(kRows)
fwd_simt_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                const float *__restrict__ u, T *__restrict__ out, float *__restrict__ neff_out,
                int Tlen, int Hq, int Hkv, float s, float alpha, float L, float beta,
                float inv_ln_L, int window) {
    __shared__ __align__(16) float Ks[kKeyTile][kHeadDim];
    __shared__ __align__(16) float Vs[kKeyTile][kHeadDim];

    const int row0 = blockIdx.x * kRows;
    const int h = blockIdx.y, b = blockIdx.z;
    const int g = h / (Hq / Hkv);
    const int i = row0 + threadIdx.x;
    const bool live = i < Tlen;

    float qr[kHeadDim];
    {
        const T *qp = q + ((static_cast<size_t>(b) * Tlen + (live ? i : 0)) * Hq + h) * kHeadDim;
#pragma unroll
        for (int d = 0; d < kHeadDim; ++d) qr[d] = live ? to_f32(qp[d]) : 0.0f;
    }
    // Causal keys 0..i; with a sliding window only the last `window` of them.
    const int lo = window > 0 ? max(0, i - window + 1) : 0;
    const int n = i + 1 - lo;
    const float c = s * length_temperature(static_cast<float>(n), alpha, L);
    const float cl2 = c * kLog2e;

    float acc[kHeadDim];
#pragma unroll
    for (int d = 0; d < kHeadDim; ++d) acc[d] = 0.0f;
    float m_ref = -INFINITY, m_raw = -INFINITY, l = 0.0f, l2 = 0.0f, s1 = 0.0f, s2 = 0.0f;

    const int kend = min(Tlen, row0 + kRows);  // keys any row of the block can see
    const int kbeg = window > 0 ? max(0, row0 - window + 1) / kKeyTile * kKeyTile : 0;
    for (int j0 = kbeg; j0 < kend; j0 += kKeyTile) {
        __syncthreads();
        for (int e = threadIdx.x; e < kKeyTile * kHeadDim; e += kRows) {
            const int jj = e / kHeadDim, d = e % kHeadDim, j = j0 + jj;
            float kv = 0.0f, vv = 0.0f;
            if (j < Tlen) {
                const size_t off = ((static_cast<size_t>(b) * Tlen + j) * Hkv + g) * kHeadDim + d;
                kv = to_f32(k[off]);
                vv = to_f32(v[off]);
            }
            Ks[jj][d] = kv;
            Vs[jj][d] = vv;
        }
        __syncthreads();
        if (!live) continue;
        const int jn = min(kKeyTile, i + 1 - j0);
        for (int jj = max(0, lo - j0); jj < jn; ++jj) {
            float sd = 0.0f;
#pragma unroll
            for (int d = 0; d < kHeadDim; d += 4) {
                const float4 kk = *reinterpret_cast<const float4 *>(&Ks[jj][d]);
                sd = fmaf(qr[d], kk.x, sd);
                sd = fmaf(qr[d + 1], kk.y, sd);
                sd = fmaf(qr[d + 2], kk.z, sd);
                sd = fmaf(qr[d + 3], kk.w, sd);
            }
            s1 += sd;
            s2 = fmaf(sd, sd, s2);
            m_raw = fmaxf(m_raw, sd);
            const float z = sd * cl2;  // logit in log2 units
            if (z > m_ref + kRescaleThreshold) {
                const float r = exp2f(m_ref - z);  // 0 on the first key
                l *= r;
                l2 *= r * r;
#pragma unroll
                for (int d = 0; d < kHeadDim; ++d) acc[d] *= r;
                m_ref = z;
            }
            const float p = exp2f(z - m_ref);
            l += p;
            l2 = fmaf(p, p, l2);
#pragma unroll
            for (int d = 0; d < kHeadDim; d += 4) {
                const float4 vv = *reinterpret_cast<const float4 *>(&Vs[jj][d]);
                acc[d] = fmaf(p, vv.x, acc[d]);
                acc[d + 1] = fmaf(p, vv.y, acc[d + 1]);
                acc[d + 2] = fmaf(p, vv.z, acc[d + 2]);
                acc[d + 3] = fmaf(p, vv.w, acc[d + 3]);
            }
        }
    }
    if (!live) return;

    float ne;
    const float mag = polar_magnitude(l, l2, m_raw, s1, s2, c, static_cast<float>(n), beta,
                                      inv_ln_L, &ne);
    float nrm = 0.0f;
#pragma unroll
    for (int d = 0; d < kHeadDim; ++d) nrm = fmaf(acc[d], acc[d], nrm);
    const float inv = 1.0f / fmaxf(sqrtf(nrm), 1e-30f);
    T *op = out + ((static_cast<size_t>(b) * Tlen + i) * Hq + h) * kHeadDim;
    const float *uh = u + static_cast<size_t>(h) * kHeadDim;
#pragma unroll
    for (int d = 0; d < kHeadDim; ++d) op[d] = from_f32<T>(fmaf(mag, uh[d], acc[d] * inv));
    if (neff_out) neff_out[(static_cast<size_t>(b) * Hq + h) * Tlen + i] = ne;
}

}  // namespace

cudaError_t launch_fwd_simt(const FwdLaunch &a) {
    dim3 grid((a.T + kRows - 1) / kRows, a.Hq, a.B);
    const float inv_ln_L = 1.0f / logf(static_cast<float>(a.L));
    if (a.dtype == POLAR_FP32) {
        fwd_simt_kernel<float><<<grid, kRows, 0, a.stream>>>(
            static_cast<const float *>(a.q), static_cast<const float *>(a.k),
            static_cast<const float *>(a.v), a.u, static_cast<float *>(a.out), a.neff, a.T, a.Hq,
            a.Hkv, a.s, a.alpha, static_cast<float>(a.L), a.beta, inv_ln_L, a.window);
    } else {
        fwd_simt_kernel<__nv_bfloat16><<<grid, kRows, 0, a.stream>>>(
            static_cast<const __nv_bfloat16 *>(a.q), static_cast<const __nv_bfloat16 *>(a.k),
            static_cast<const __nv_bfloat16 *>(a.v), a.u, static_cast<__nv_bfloat16 *>(a.out),
            a.neff, a.T, a.Hq, a.Hkv, a.s, a.alpha, static_cast<float>(a.L), a.beta, inv_ln_L,
            a.window);
    }
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace polar
