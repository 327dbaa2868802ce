// bwd_simt.cu -- backward of the causal Polar Attention prefill (CUDA cores).
//
// Given g = dL/dout for every row, the gradients dL/dq, dL/dk, dL/dv and
// dL/du of the step out = content + gate * tanh(ln n_eff / ln L) * u_h (ATMA
// technical summary, section 2.1; the training use of the fused kernel of
// section 2.2).  With w_j = 2^(cl2 S_j - ref) for the row's own reference,
// l = sum w, l2 = sum w^2, A = sum w_j v_j, content = A/|A|, T = tanh(ln n_eff
// / ln L), the chain rule gives, per row:
//   du_h   += gate * T * g
//   gamma   = <g, u_h>;  dgate = gamma T;  dT = gamma gate
//   dn_eff  = dT (1 - T^2) / (n_eff ln L)      (0 where n_eff is clamped)
//   dl      = 2 (l/l2) dn_eff;   dl2 = -(l/l2)^2 dn_eff
//   dA      = (g - content <content, g>) / |A|
//   dm      = beta gate (1 - gate) dgate;   dmu = -dm;   dsigma = -dm sqrt(2 ln n)
//   dz_j    = w_j (dl + 2 dl2 w_j + <dA, v_j>) + dmu/n + dsigma (z_j - mu)/(n sigma)
//             + [j = first argmax] dm
//   dS_j    = c dz_j;  dq += dS_j k_j;  dk_j += dS_j q;  dv_j += w_j dA.
// (w, l, l2 and A may share any reference: content and n_eff are scale-free.)
//
// Four launches.  For fp32 inputs they run on the CUDA cores in fp32 (below);
// for bf16 inputs pass 1 runs its contractions on mma.sync tensor-core tiles
// (bwd_rows_mma_kernel) and passes 2-3 are the tcgen05/TMEM kernels of
// bwd_tc.cu, which read the rows pass's compact coefficient records:
//  1. rows: one thread per query row recomputes the row's forward state
//     (streaming, as the CUDA-core prefill does, plus the first argmax) and
//     writes the row's coefficients: dA, the reference and scales, dl, dl2,
//     the constant and S-linear terms of dz, dm, the argmax and the window's
//     first key, and gate * T for du.
//  2. dk, dv: two threads per key (one per half of the 64 components) keep
//     the key's k, v and its dk, dv in registers while the rows that see it
//     stream through shared memory; every query head of the group adds in.
//  3. dq: two threads per query row keep q, dA and dq in registers while the
//     keys stream through shared memory.
//  4. du: per head, the sum over rows of gate * T * g.
// Each kernel recomputes S_j with the same fp32 summation order, so the argmax
// test is an index comparison.
#include <type_traits>

#include "bwd_coef.cuh"
#include "polar_common.cuh"
#include "polar_internal.h"

namespace polar {
namespace {

constexpr int kRowsB0 = 128;  // rows per block of the rows kernel
constexpr int kKeyTile = 64;  // keys per shared-memory stage
constexpr int kRowStage = 32; // rows per shared-memory stage of the dk/dv kernel

// Per-row coefficient record (fp32 words).
constexpr int kRecDA = 0;      // dA[64]
constexpr int kRecRef = 64;    // exponent reference (log2 units)
constexpr int kRecCl2 = 65;    // c * log2(e)
constexpr int kRecC = 66;      // c
constexpr int kRecDl = 67;
constexpr int kRecDl2 = 68;
constexpr int kRecCmu = 69;    // constant term of dz
constexpr int kRecCsS = 70;    // coefficient of S in dz
constexpr int kRecDm = 71;     // argmax term
constexpr int kRecJmax = 72;   // first argmax key (int bits)
constexpr int kRecLo = 73;     // first visible key (int bits)
constexpr int kRecGT = 74;     // gate * T
constexpr int kRecWords = 80;

struct BwdArgs {
    const float *u;
    float *rec;      // fp32 inputs: [B][Hq][T][kRecWords]
    float *du_part;  // [B * row blocks][Hq][64]: per-block sums of gate * T * g
    float *coef;     // bf16 inputs: [B][Hq][Tpad][kBwdCoefWords] (BwdCoef layout)
    __nv_bfloat16 *dab;  // bf16 inputs: [B][Hq][Tpad][64], dA rounded to bf16
    int B, T, Tpad, Hq, Hkv, window;
    float s, alpha, L, beta, inv_ln_L;
};

// ------------------------------------------------------------------ rows ---
template <typename T>
__global__ void __launch_bounds__(kRowsB0)
bwd_rows_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                const T *__restrict__ gout, const BwdArgs a) {
    __shared__ __align__(16) float Ks[kKeyTile][kHeadDim];
    __shared__ __align__(16) float Vs[kKeyTile][kHeadDim];
    const int Tlen = a.T;
    const int row0 = blockIdx.x * kRowsB0;
    const int h = blockIdx.y, b = blockIdx.z;
    const int g = h / (a.Hq / a.Hkv);
    const int i = row0 + threadIdx.x;
    const bool live = i < Tlen;

    float qr[kHeadDim];
    {
        const T *qp = q + ((static_cast<size_t>(b) * Tlen + (live ? i : 0)) * a.Hq + h) * kHeadDim;
#pragma unroll
        for (int d = 0; d < kHeadDim; ++d) qr[d] = live ? to_f32(qp[d]) : 0.0f;
    }
    const int lo = a.window > 0 ? max(0, i - a.window + 1) : 0;
    const int n = i + 1 - lo;
    const float c = a.s * length_temperature(static_cast<float>(n), a.alpha, a.L);
    const float cl2 = c * kLog2e;

    float acc[kHeadDim];
#pragma unroll
    for (int d = 0; d < kHeadDim; ++d) acc[d] = 0.0f;
    float m_ref = -INFINITY, m_raw = -INFINITY, l = 0.0f, l2 = 0.0f, s1 = 0.0f, s2 = 0.0f;
    int jmax = lo;

    const int kend = min(Tlen, row0 + kRowsB0);
    const int kbeg = a.window > 0 ? max(0, row0 - a.window + 1) / kKeyTile * kKeyTile : 0;
    for (int j0 = kbeg; j0 < kend; j0 += kKeyTile) {
        __syncthreads();
        for (int e = threadIdx.x; e < kKeyTile * kHeadDim; e += kRowsB0) {
            const int jj = e / kHeadDim, d = e % kHeadDim, j = j0 + jj;
            float kv = 0.0f, vv = 0.0f;
            if (j < Tlen) {
                const size_t off = ((static_cast<size_t>(b) * Tlen + j) * a.Hkv + g) * kHeadDim + d;
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
            if (sd > m_raw) {  // strict: the first index of the max
                m_raw = sd;
                jmax = j0 + jj;
            }
            const float z = sd * cl2;
            if (z > m_ref + kRescaleThreshold) {
                const float r = exp2f(m_ref - z);
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
    const float nf = static_cast<float>(live ? n : 1);
    const float mean_s = s1 / nf;
    const float sig_s = sqrtf(fmaxf(s2 / nf - mean_s * mean_s, 0.0f));
    const float mu = c * mean_s, sigma = c * sig_s;
    const float kn = sqrtf(2.0f * logf(nf));
    const float z0 = mu + sigma * kn;
    const float gate = 1.0f / (1.0f + expf(-a.beta * (c * m_raw - z0)));
    const float ne_raw = (l * l) / l2;
    const float ne = fminf(fmaxf(ne_raw, 1.0f), nf);
    const bool clamped = ne != ne_raw;
    const float Tm = tanhf(logf(ne) * a.inv_ln_L);
    float nrm = 0.0f;
#pragma unroll
    for (int d = 0; d < kHeadDim; ++d) nrm = fmaf(acc[d], acc[d], nrm);
    const float an = fmaxf(sqrtf(nrm), 1e-30f);
    const float inv_an = 1.0f / an;

    const T *gp = gout + ((static_cast<size_t>(b) * Tlen + (live ? i : 0)) * a.Hq + h) * kHeadDim;
    const float *uh = a.u + static_cast<size_t>(h) * kHeadDim;
    float gamma = 0.0f, cg = 0.0f;
#pragma unroll
    for (int d = 0; d < kHeadDim; ++d) {
        const float gd = live ? to_f32(gp[d]) : 0.0f;
        qr[d] = gd;  // q is no longer needed: reuse the registers for g
        gamma = fmaf(gd, uh[d], gamma);
        cg = fmaf(acc[d] * inv_an, gd, cg);
    }
    const float dgate = gamma * Tm, dT = gamma * gate;
    const float dneff = clamped ? 0.0f : dT * (1.0f - Tm * Tm) * a.inv_ln_L / ne;
    const float dl = 2.0f * dneff * l / l2;
    const float dl2 = -dneff * (l / l2) * (l / l2);
    const float dm = a.beta * gate * (1.0f - gate) * dgate;
    const float dmu = -dm, dsigma = -dm * kn;
    const float cmu = dmu / nf - (sigma > 0.0f ? dsigma * mu / (nf * sigma) : 0.0f);
    const float csS = sigma > 0.0f ? dsigma * c / (nf * sigma) : 0.0f;

    // du: this block's sum over its rows of gate * T * g, through the (now
    // free) key stages; rows past the end add nothing.
    __syncthreads();
    float(*red)[kHeadDim] = reinterpret_cast<float(*)[kHeadDim]>(&Ks[0][0]);  // [128][64]
    static_assert(sizeof(Ks) + sizeof(Vs) >= kRowsB0 * kHeadDim * sizeof(float), "stage too small");
    const float gt = live ? gate * Tm : 0.0f;
#pragma unroll
    for (int d = 0; d < kHeadDim; ++d) red[threadIdx.x][(d + threadIdx.x) & (kHeadDim - 1)] = gt * qr[d];
    __syncthreads();
    if (threadIdx.x < kHeadDim) {
        const int d = threadIdx.x;
        float sum = 0.0f;
        for (int t = 0; t < kRowsB0; ++t) sum += red[t][(d + t) & (kHeadDim - 1)];
        a.du_part[((static_cast<size_t>(b) * gridDim.x + blockIdx.x) * a.Hq + h) * kHeadDim + d] = sum;
    }
    if (!live) return;

    float *rec = a.rec + ((static_cast<size_t>(b) * a.Hq + h) * Tlen + i) * kRecWords;
#pragma unroll
    for (int d = 0; d < kHeadDim; d += 4)
        *reinterpret_cast<float4 *>(rec + kRecDA + d) =
            make_float4((qr[d] - acc[d] * inv_an * cg) * inv_an,
                        (qr[d + 1] - acc[d + 1] * inv_an * cg) * inv_an,
                        (qr[d + 2] - acc[d + 2] * inv_an * cg) * inv_an,
                        (qr[d + 3] - acc[d + 3] * inv_an * cg) * inv_an);
    *reinterpret_cast<float4 *>(rec + 64) = make_float4(m_ref, cl2, c, dl);
    *reinterpret_cast<float4 *>(rec + 68) = make_float4(dl2, cmu, csS, dm);
    static_assert(kRecJmax == 72 && kRecLo == 73 && kRecGT == 74, "record layout");
    *reinterpret_cast<float4 *>(rec + kRecJmax) =
        make_float4(__int_as_float(jmax), __int_as_float(lo), gate * Tm, 0.0f);
}

// The scalars of a row's record.
struct RowCoef {
    float ref, cl2, c, dl, dl2, cmu, csS, dm;
    int jmax, lo;
};

__device__ __forceinline__ RowCoef load_coef(const float *rc) {
    RowCoef r;
    r.ref = rc[kRecRef]; r.cl2 = rc[kRecCl2]; r.c = rc[kRecC]; r.dl = rc[kRecDl];
    r.dl2 = rc[kRecDl2]; r.cmu = rc[kRecCmu]; r.csS = rc[kRecCsS]; r.dm = rc[kRecDm];
    r.jmax = __float_as_int(rc[kRecJmax]);
    r.lo = __float_as_int(rc[kRecLo]);
    return r;
}

// dS_j = c dz_j for one (row, key) pair from the row's coefficients and the
// pair's two dot products S = <q, k_j>, av = <dA, v_j>; w = the weight.
__device__ __forceinline__ float pair_ds(const RowCoef &r, float S, float av, int j, float &w) {
    w = exp2f(fmaf(S, r.cl2, -r.ref));
    float dz = fmaf(w, fmaf(2.0f * r.dl2, w, r.dl + av), fmaf(r.csS, S, r.cmu));
    if (j == r.jmax) dz += r.dm;
    return dz * r.c;
}

// ----------------------------------------------------------------- dk, dv ---
template <typename T>
__global__ void __launch_bounds__(128)
bwd_dkdv_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                float *__restrict__ dk, float *__restrict__ dv, const BwdArgs a) {
    __shared__ __align__(16) float Qs[kRowStage][kHeadDim];
    __shared__ __align__(16) float Rs[kRowStage][kRecWords];
    const int Tlen = a.T, G = a.Hq / a.Hkv;
    const int key0 = blockIdx.x * kKeyTile, g = blockIdx.y, b = blockIdx.z;
    const int j = key0 + (threadIdx.x >> 1), half = threadIdx.x & 1;
    const bool jlive = j < Tlen;
    float kr[32], vr[32], dkr[32], dvr[32];
    {
        const size_t off = ((static_cast<size_t>(b) * Tlen + (jlive ? j : 0)) * a.Hkv + g) * kHeadDim +
                           32 * half;
#pragma unroll
        for (int d = 0; d < 32; ++d) {
            kr[d] = jlive ? to_f32(k[off + d]) : 0.0f;
            vr[d] = jlive ? to_f32(v[off + d]) : 0.0f;
            dkr[d] = dvr[d] = 0.0f;
        }
    }
    // Rows that see any key of the tile: key0 .. key0 + 63 + window - 1.
    const int iend = a.window > 0 ? min(Tlen, key0 + kKeyTile - 1 + a.window) : Tlen;
    for (int hh = 0; hh < G; ++hh) {
        const int h = g * G + hh;
        for (int i0 = key0; i0 < iend; i0 += kRowStage) {
            __syncthreads();
            for (int e = threadIdx.x; e < kRowStage * kHeadDim; e += 128) {
                const int rr = e / kHeadDim, d = e % kHeadDim, i = i0 + rr;
                Qs[rr][d] = i < Tlen ? to_f32(q[((static_cast<size_t>(b) * Tlen + i) * a.Hq + h) *
                                                    kHeadDim + d])
                                     : 0.0f;
            }
            for (int e = threadIdx.x; e < kRowStage * kRecWords; e += 128) {
                const int rr = e / kRecWords, wd = e % kRecWords, i = i0 + rr;
                Rs[rr][wd] = i < Tlen ? a.rec[((static_cast<size_t>(b) * a.Hq + h) * Tlen + i) *
                                                  kRecWords + wd]
                                      : 0.0f;
            }
            __syncthreads();
            const int nr = min(kRowStage, iend - i0);
            for (int rr = 0; rr < nr; ++rr) {
                const int i = i0 + rr;
                const float *rc = Rs[rr];
                float sp = 0.0f, ap = 0.0f;
#pragma unroll
                for (int d = 0; d < 32; d += 4) {
                    const float4 qq = *reinterpret_cast<const float4 *>(&Qs[rr][32 * half + d]);
                    const float4 da = *reinterpret_cast<const float4 *>(&rc[kRecDA + 32 * half + d]);
                    sp = fmaf(qq.x, kr[d], sp);
                    sp = fmaf(qq.y, kr[d + 1], sp);
                    sp = fmaf(qq.z, kr[d + 2], sp);
                    sp = fmaf(qq.w, kr[d + 3], sp);
                    ap = fmaf(da.x, vr[d], ap);
                    ap = fmaf(da.y, vr[d + 1], ap);
                    ap = fmaf(da.z, vr[d + 2], ap);
                    ap = fmaf(da.w, vr[d + 3], ap);
                }
                // Lower half first, so that both threads of a key sum in the same order.
                const float so = __shfl_xor_sync(0xffffffffu, sp, 1);
                const float ao = __shfl_xor_sync(0xffffffffu, ap, 1);
                const float S = half ? so + sp : sp + so;
                const float av = half ? ao + ap : ap + ao;
                const RowCoef cf = load_coef(rc);
                const bool vis = jlive && j <= i && j >= cf.lo;
                float w;
                const float dS = pair_ds(cf, S, av, j, w);
                const float ds = vis ? dS : 0.0f, ww = vis ? w : 0.0f;
#pragma unroll
                for (int d = 0; d < 32; d += 4) {
                    const float4 qq = *reinterpret_cast<const float4 *>(&Qs[rr][32 * half + d]);
                    const float4 da = *reinterpret_cast<const float4 *>(&rc[kRecDA + 32 * half + d]);
                    dkr[d] = fmaf(ds, qq.x, dkr[d]);
                    dkr[d + 1] = fmaf(ds, qq.y, dkr[d + 1]);
                    dkr[d + 2] = fmaf(ds, qq.z, dkr[d + 2]);
                    dkr[d + 3] = fmaf(ds, qq.w, dkr[d + 3]);
                    dvr[d] = fmaf(ww, da.x, dvr[d]);
                    dvr[d + 1] = fmaf(ww, da.y, dvr[d + 1]);
                    dvr[d + 2] = fmaf(ww, da.z, dvr[d + 2]);
                    dvr[d + 3] = fmaf(ww, da.w, dvr[d + 3]);
                }
            }
        }
    }
    if (!jlive) return;
    const size_t off = ((static_cast<size_t>(b) * Tlen + j) * a.Hkv + g) * kHeadDim + 32 * half;
#pragma unroll
    for (int d = 0; d < 32; d += 4) {
        *reinterpret_cast<float4 *>(dk + off + d) = make_float4(dkr[d], dkr[d + 1], dkr[d + 2], dkr[d + 3]);
        *reinterpret_cast<float4 *>(dv + off + d) = make_float4(dvr[d], dvr[d + 1], dvr[d + 2], dvr[d + 3]);
    }
}

// -------------------------------------------------------------------- dq ---
template <typename T>
__global__ void __launch_bounds__(128)
bwd_dq_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
              float *__restrict__ dq, const BwdArgs a) {
    __shared__ __align__(16) float Ks[kKeyTile][kHeadDim];
    __shared__ __align__(16) float Vs[kKeyTile][kHeadDim];
    const int Tlen = a.T;
    const int row0 = blockIdx.x * kKeyTile, h = blockIdx.y, b = blockIdx.z;
    const int g = h / (a.Hq / a.Hkv);
    const int i = row0 + (threadIdx.x >> 1), half = threadIdx.x & 1;
    const bool live = i < Tlen;
    float qr[32], dar[32], dqr[32];
    RowCoef cf;
    {
        const size_t qo = ((static_cast<size_t>(b) * Tlen + (live ? i : 0)) * a.Hq + h) * kHeadDim + 32 * half;
        const float *rp = a.rec + ((static_cast<size_t>(b) * a.Hq + h) * Tlen + (live ? i : 0)) * kRecWords;
#pragma unroll
        for (int d = 0; d < 32; ++d) {
            qr[d] = live ? to_f32(q[qo + d]) : 0.0f;
            dar[d] = live ? rp[kRecDA + 32 * half + d] : 0.0f;
            dqr[d] = 0.0f;
        }
        cf = load_coef(rp);  // row 0's record stands in for a row past the end
    }
    const int lo = cf.lo;
    const int kend = min(Tlen, row0 + kKeyTile);
    const int kbeg = a.window > 0 ? max(0, row0 - a.window + 1) / kKeyTile * kKeyTile : 0;
    for (int j0 = kbeg; j0 < kend; j0 += kKeyTile) {
        __syncthreads();
        for (int e = threadIdx.x; e < kKeyTile * kHeadDim; e += 128) {
            const int jj = e / kHeadDim, d = e % kHeadDim, j = j0 + jj;
            float kv = 0.0f, vv = 0.0f;
            if (j < Tlen) {
                const size_t off = ((static_cast<size_t>(b) * Tlen + j) * a.Hkv + g) * kHeadDim + d;
                kv = to_f32(k[off]);
                vv = to_f32(v[off]);
            }
            Ks[jj][d] = kv;
            Vs[jj][d] = vv;
        }
        __syncthreads();
        const int jn = min(kKeyTile, kend - j0);
        for (int jj = 0; jj < jn; ++jj) {
            const int j = j0 + jj;
            float sp = 0.0f, ap = 0.0f;
#pragma unroll
            for (int d = 0; d < 32; d += 4) {
                const float4 kk = *reinterpret_cast<const float4 *>(&Ks[jj][32 * half + d]);
                const float4 vv = *reinterpret_cast<const float4 *>(&Vs[jj][32 * half + d]);
                sp = fmaf(qr[d], kk.x, sp);
                sp = fmaf(qr[d + 1], kk.y, sp);
                sp = fmaf(qr[d + 2], kk.z, sp);
                sp = fmaf(qr[d + 3], kk.w, sp);
                ap = fmaf(dar[d], vv.x, ap);
                ap = fmaf(dar[d + 1], vv.y, ap);
                ap = fmaf(dar[d + 2], vv.z, ap);
                ap = fmaf(dar[d + 3], vv.w, ap);
            }
            const float so = __shfl_xor_sync(0xffffffffu, sp, 1);
            const float ao = __shfl_xor_sync(0xffffffffu, ap, 1);
            const float S = half ? so + sp : sp + so;
            const float av = half ? ao + ap : ap + ao;
            const bool vis = live && j <= i && j >= lo;
            float w;
            const float dS = pair_ds(cf, S, av, j, w);
            const float ds = vis ? dS : 0.0f;
#pragma unroll
            for (int d = 0; d < 32; d += 4) {
                const float4 kk = *reinterpret_cast<const float4 *>(&Ks[jj][32 * half + d]);
                dqr[d] = fmaf(ds, kk.x, dqr[d]);
                dqr[d + 1] = fmaf(ds, kk.y, dqr[d + 1]);
                dqr[d + 2] = fmaf(ds, kk.z, dqr[d + 2]);
                dqr[d + 3] = fmaf(ds, kk.w, dqr[d + 3]);
            }
        }
    }
    if (!live) return;
    const size_t qo = ((static_cast<size_t>(b) * Tlen + i) * a.Hq + h) * kHeadDim + 32 * half;
#pragma unroll
    for (int d = 0; d < 32; d += 4)
        *reinterpret_cast<float4 *>(dq + qo + d) = make_float4(dqr[d], dqr[d + 1], dqr[d + 2], dqr[d + 3]);
}


// ------------------------------------------- tensor-core (mma.sync) kernels ---
// For bf16 inputs the contractions of the dk/dv and dq passes run on the
// tensor cores (m16n8k16, bf16 in, fp32 accumulate): the scores and <dA, v>
// are recomputed as tile products, dz is formed in the accumulator fragments
// and re-packed as the A operand of the gradient products (dA, dS and w are
// rounded to bf16 for those products).  Tiles of 64 rows x 64 dims live in
// shared memory with a 144-byte row pitch, so that the ldmatrix reads are free
// of bank conflicts.
constexpr int kPitch = 72;  // bf16 per padded row (144 bytes)

__device__ __forceinline__ void ldsm4(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm4t(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pk2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// A fragments (16 rows x 64, 4 k-steps) of rows r0 + lane/4 and r0 + lane/4 + 8
// of a bf16 [*, stride] matrix in global memory; rows at or past `rows` are 0.
__device__ __forceinline__ void load_a_rows(const __nv_bfloat16 *base, size_t stride, int r0,
                                            int rows, uint32_t (&fa)[4][4]) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const int ra = r0 + g, rb = r0 + g + 8;
    const uint32_t *pa = reinterpret_cast<const uint32_t *>(base + static_cast<size_t>(ra < rows ? ra : 0) * stride);
    const uint32_t *pb = reinterpret_cast<const uint32_t *>(base + static_cast<size_t>(rb < rows ? rb : 0) * stride);
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
        fa[ks][0] = ra < rows ? pa[8 * ks + t] : 0u;
        fa[ks][1] = rb < rows ? pb[8 * ks + t] : 0u;
        fa[ks][2] = ra < rows ? pa[8 * ks + 4 + t] : 0u;
        fa[ks][3] = rb < rows ? pb[8 * ks + 4 + t] : 0u;
    }
}

// Copy 64 rows (64 bf16 each) into a padded shared tile; rows past `valid` are 0.
__device__ __forceinline__ void stage_rows(__nv_bfloat16 (*dst)[kPitch], const __nv_bfloat16 *src,
                                           size_t stride, int valid) {
    for (int e = threadIdx.x; e < 64 * 8; e += blockDim.x) {
        const int r = e >> 3, c = e & 7;
        uint4 val = make_uint4(0u, 0u, 0u, 0u);
        if (r < valid) val = *reinterpret_cast<const uint4 *>(src + static_cast<size_t>(r) * stride + 8 * c);
        *reinterpret_cast<uint4 *>(&dst[r][8 * c]) = val;
    }
}

// S-like products of a warp's 16 A rows with 64 shared rows: out[nt] holds
// columns 8nt .. 8nt+7 (the shared rows), i.e. sum over the 64 dims of
// A[row][d] * M[col][d].
__device__ __forceinline__ void rows_times_tile(const uint32_t (&fa)[4][4], uint32_t tile,
                                                float (&out)[8][4]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
        out[nt][0] = out[nt][1] = out[nt][2] = out[nt][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {  // 32 dims per ldmatrix.x4
            uint32_t b[4];
            ldsm4(tile + ((8 * nt + (lane & 7)) * kPitch + 32 * kk + 8 * (lane >> 3)) * 2, b);
            mma16816(out[nt], fa[2 * kk], b[0], b[1]);
            mma16816(out[nt], fa[2 * kk + 1], b[2], b[3]);
        }
    }
}

// acc[nt] += P (16 x 64, as 4 k-steps of A fragments) times the 64 x 64 shared
// tile (rows = the k dimension, columns = the 64 dims): columns 8nt .. 8nt+7.
__device__ __forceinline__ void frag_times_tile(const uint32_t (&pa)[4][4], uint32_t tile,
                                                float (&acc)[8][4]) {
    const int lane = threadIdx.x & 31, mi = lane >> 3;
#pragma unroll
    for (int ks = 0; ks < 4; ++ks)
#pragma unroll
        for (int p = 0; p < 4; ++p) {  // dims 16p .. 16p+15: two n-tiles
            uint32_t b[4];
            ldsm4t(tile + ((16 * ks + (lane & 7) + 8 * (mi & 1)) * kPitch + 16 * p + 8 * (mi >> 1)) * 2, b);
            mma16816(acc[2 * p], pa[ks], b[0], b[1]);
            mma16816(acc[2 * p + 1], pa[ks], b[2], b[3]);
        }
}


// Rows pass for bf16 inputs on the tensor cores: a warp owns 16 query rows
// (two per lane: rows lane/4 and lane/4 + 8); key blocks of 64 stream through
// shared memory.  S = Q K^T and O += P V are tile products; the row statistics
// (first argmax, S1, S2, l, l2 under a lazy reference) come from the
// accumulator fragments with quad shuffles.  The epilogue writes the same
// record as bwd_rows_kernel, and a du partial per 64-row block.
__global__ void __launch_bounds__(128)
bwd_rows_mma_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
                    const __nv_bfloat16 *__restrict__ v, const __nv_bfloat16 *__restrict__ gout,
                    const BwdArgs a) {
    __shared__ __align__(16) __nv_bfloat16 Ks[64][kPitch];
    __shared__ __align__(16) __nv_bfloat16 Vs[64][kPitch];
    __shared__ float red[4][kHeadDim];
    const int Tlen = a.T, G = a.Hq / a.Hkv;
    const int row0 = blockIdx.x * 64, h = blockIdx.y, b = blockIdx.z, g = h / G;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, gq = lane >> 2, tq = lane & 3;
    const int r0 = row0 + 16 * warp;
    const size_t qstride = static_cast<size_t>(a.Hq) * kHeadDim;
    const size_t kstride = static_cast<size_t>(a.Hkv) * kHeadDim;
    uint32_t qa[4][4];
    load_a_rows(q + (static_cast<size_t>(b) * Tlen * a.Hq + h) * kHeadDim, qstride, r0, Tlen, qa);
    int rowi[2], lo[2];
    float cl2[2], cc[2];
    float m_ref[2], m_raw[2], l[2], l2[2], s1[2], s2[2];
    int jmax[2];
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
        const int i = r0 + gq + 8 * hr;
        rowi[hr] = i;
        lo[hr] = a.window > 0 ? max(0, i - a.window + 1) : 0;
        const float n = static_cast<float>(i + 1 - lo[hr]);
        cc[hr] = a.s * length_temperature(n, a.alpha, a.L);
        cl2[hr] = cc[hr] * kLog2e;
        m_ref[hr] = m_raw[hr] = -INFINITY;
        l[hr] = l2[hr] = s1[hr] = s2[hr] = 0.f;
        jmax[hr] = lo[hr];
    }
    float acc[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
    const uint32_t ks_addr = smem_u32(&Ks[0][0]), vs_addr = smem_u32(&Vs[0][0]);
    // A block past the end only pads the records to a multiple of 128 rows.
    const int kend = row0 < Tlen ? min(Tlen, row0 + 64) : 0;
    const int kbeg = a.window > 0 ? max(0, row0 - a.window + 1) / 64 * 64 : 0;
    for (int j0 = kbeg; j0 < kend; j0 += 64) {
        __syncthreads();
        stage_rows(Ks, k + ((static_cast<size_t>(b) * Tlen + j0) * a.Hkv + g) * kHeadDim, kstride, Tlen - j0);
        stage_rows(Vs, v + ((static_cast<size_t>(b) * Tlen + j0) * a.Hkv + g) * kHeadDim, kstride, Tlen - j0);
        __syncthreads();
        float sc[8][4];
        rows_times_tile(qa, ks_addr, sc);
        float pw[8][4];
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
            const int i = rowi[hr];
            float tmax = -INFINITY, ts1 = 0.f, ts2 = 0.f;
            int tidx = 0x7fffffff;
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int j = j0 + 8 * nt + 2 * tq + e;
                    const bool vis = i < Tlen && j <= i && j >= lo[hr];
                    const float x = sc[nt][2 * hr + e];
                    if (vis && x > tmax) { tmax = x; tidx = j; }  // columns ascend within a lane
                    ts1 += vis ? x : 0.f;
                    ts2 += vis ? x * x : 0.f;
                }
#pragma unroll
            for (int off = 1; off <= 2; off <<= 1) {
                const float ov = __shfl_xor_sync(0xffffffffu, tmax, off);
                const int oi = __shfl_xor_sync(0xffffffffu, tidx, off);
                if (ov > tmax || (ov == tmax && oi < tidx)) { tmax = ov; tidx = oi; }
            }
            if (tmax > m_raw[hr]) { m_raw[hr] = tmax; jmax[hr] = tidx; }  // strict: first index
            s1[hr] += ts1;
            s2[hr] += ts2;
            const float zmax = tmax * cl2[hr];
            if (zmax > m_ref[hr] + kRescaleThreshold) {  // uniform over the quad
                const float r = exp2f(m_ref[hr] - zmax);
                l[hr] *= r;
                l2[hr] *= r * r;
#pragma unroll
                for (int nt = 0; nt < 8; ++nt) {
                    acc[nt][2 * hr] *= r;
                    acc[nt][2 * hr + 1] *= r;
                }
                m_ref[hr] = zmax;
            }
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int j = j0 + 8 * nt + 2 * tq + e;
                    const bool vis = i < Tlen && j <= i && j >= lo[hr];
                    const float pp = vis ? exp2f(fmaf(sc[nt][2 * hr + e], cl2[hr], -m_ref[hr])) : 0.f;
                    pw[nt][2 * hr + e] = pp;
                    l[hr] += pp;
                    l2[hr] = fmaf(pp, pp, l2[hr]);
                }
        }
        uint32_t pa[4][4];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
            pa[nt >> 1][(nt & 1) * 2] = pk2(pw[nt][0], pw[nt][1]);
            pa[nt >> 1][(nt & 1) * 2 + 1] = pk2(pw[nt][2], pw[nt][3]);
        }
        frag_times_tile(pa, vs_addr, acc);  // O += P V
    }

    // Epilogue per row: quad sums of the partial statistics and dot products.
    float dupart[8][2];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) dupart[nt][0] = dupart[nt][1] = 0.f;
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
        const int i = rowi[hr];
        const bool live = i < Tlen;
        float gr[8][2], nrm = 0.f, gamma = 0.f, cgr = 0.f;
        const __nv_bfloat16 *gp = gout + ((static_cast<size_t>(b) * Tlen + (live ? i : 0)) * a.Hq + h) * kHeadDim;
        const float *uh = a.u + static_cast<size_t>(h) * kHeadDim;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
            const int d = 8 * nt + 2 * tq;
            const __nv_bfloat162 gg = *reinterpret_cast<const __nv_bfloat162 *>(gp + d);
            gr[nt][0] = live ? __low2float(gg) : 0.f;
            gr[nt][1] = live ? __high2float(gg) : 0.f;
            const float o0 = acc[nt][2 * hr], o1 = acc[nt][2 * hr + 1];
            nrm = fmaf(o0, o0, fmaf(o1, o1, nrm));
            gamma = fmaf(gr[nt][0], uh[d], fmaf(gr[nt][1], uh[d + 1], gamma));
            cgr = fmaf(o0, gr[nt][0], fmaf(o1, gr[nt][1], cgr));
        }
        float ll = l[hr], ll2 = l2[hr], ss1 = s1[hr], ss2 = s2[hr];
#pragma unroll
        for (int off = 1; off <= 2; off <<= 1) {
            nrm += __shfl_xor_sync(0xffffffffu, nrm, off);
            gamma += __shfl_xor_sync(0xffffffffu, gamma, off);
            cgr += __shfl_xor_sync(0xffffffffu, cgr, off);
            ll += __shfl_xor_sync(0xffffffffu, ll, off);
            ll2 += __shfl_xor_sync(0xffffffffu, ll2, off);
            ss1 += __shfl_xor_sync(0xffffffffu, ss1, off);
            ss2 += __shfl_xor_sync(0xffffffffu, ss2, off);
        }
        const float nf = static_cast<float>(live ? i + 1 - lo[hr] : 1);
        const float c = cc[hr];
        const float mean_s = ss1 / nf;
        const float sig_s = sqrtf(fmaxf(ss2 / nf - mean_s * mean_s, 0.0f));
        const float mu = c * mean_s, sigma = c * sig_s;
        const float kn = sqrtf(2.0f * logf(nf));
        const float z0 = mu + sigma * kn;
        const float gate = 1.0f / (1.0f + expf(-a.beta * (c * m_raw[hr] - z0)));
        const float ne_raw = (ll * ll) / ll2;
        const float ne = fminf(fmaxf(ne_raw, 1.0f), nf);
        const bool clamped = ne != ne_raw;
        const float Tm = tanhf(logf(ne) * a.inv_ln_L);
        const float an = fmaxf(sqrtf(nrm), 1e-30f), inv_an = 1.0f / an;
        const float cg = cgr * inv_an;  // <content, g>
        const float dgate = gamma * Tm, dT = gamma * gate;
        const float dneff = clamped ? 0.0f : dT * (1.0f - Tm * Tm) * a.inv_ln_L / ne;
        const float dl = 2.0f * dneff * ll / ll2;
        const float dl2 = -dneff * (ll / ll2) * (ll / ll2);
        const float dm = a.beta * gate * (1.0f - gate) * dgate;
        const float dmu = -dm, dsigma = -dm * kn;
        const float cmu = dmu / nf - (sigma > 0.0f ? dsigma * mu / (nf * sigma) : 0.0f);
        const float csS = sigma > 0.0f ? dsigma * c / (nf * sigma) : 0.0f;
        const float gt = live ? gate * Tm : 0.0f;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
            dupart[nt][0] = fmaf(gt, gr[nt][0], dupart[nt][0]);
            dupart[nt][1] = fmaf(gt, gr[nt][1], dupart[nt][1]);
        }
        // dA rounded to bf16 and the row's compact coefficient record (rows past
        // the end: zero dA, and cl2 = c = 0 with nref = -inf, so that their
        // weights and dS vanish in the later passes without masks).
        const size_t rrow = (static_cast<size_t>(b) * a.Hq + h) * a.Tpad + i;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
            const int d = 8 * nt + 2 * tq;
            const float o0 = acc[nt][2 * hr] * inv_an, o1 = acc[nt][2 * hr + 1] * inv_an;
            const float da0 = live ? (gr[nt][0] - o0 * cg) * inv_an : 0.f;
            const float da1 = live ? (gr[nt][1] - o1 * cg) * inv_an : 0.f;
            *reinterpret_cast<uint32_t *>(a.dab + rrow * kHeadDim + d) = pk2(da0, da1);
        }
        if (tq == 0) {
            float4 *cr = reinterpret_cast<float4 *>(a.coef + rrow * kBwdCoefWords);
            if (live) {
                cr[0] = make_float4(cl2[hr], -m_ref[hr], c, c * dl);
                cr[1] = make_float4(2.0f * c * dl2, c * csS, c * cmu, c * dm);
                cr[2] = make_float4(__int_as_float(jmax[hr]), __int_as_float(lo[hr]), gt, 0.f);
            } else {
                cr[0] = make_float4(0.f, -INFINITY, 0.f, 0.f);
                cr[1] = make_float4(0.f, 0.f, 0.f, 0.f);
                cr[2] = make_float4(__int_as_float(-1), __int_as_float(0), 0.f, 0.f);
            }
            cr[3] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    // du: sum over the warp's 16 rows (lanes of equal tq), then over the warps.
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            float x = dupart[nt][e];
            x += __shfl_xor_sync(0xffffffffu, x, 4);
            x += __shfl_xor_sync(0xffffffffu, x, 8);
            x += __shfl_xor_sync(0xffffffffu, x, 16);
            if (gq == 0) red[warp][8 * nt + 2 * tq + e] = x;
        }
    __syncthreads();
    if (threadIdx.x < kHeadDim) {
        const int d = threadIdx.x;
        a.du_part[((static_cast<size_t>(b) * gridDim.x + blockIdx.x) * a.Hq + h) * kHeadDim + d] =
            (red[0][d] + red[1][d]) + (red[2][d] + red[3][d]);
    }
}

// -------------------------------------------------------------------- du ---
// du partials of one 16-row block per (block, batch), all heads: the sum over
// its rows of gate*T (from the coefficient records) times the upstream
// gradient.  Used after the tensor-core rows pass, which writes no du
// partials.  Each thread owns 8 consecutive elements of a row's [Hq, 64] slab
// of dout and issues its 16 rows' 16-byte loads together.
constexpr int kDuRows = 16;
__global__ void __launch_bounds__(128)
bwd_du_part_kernel(const __nv_bfloat16 *__restrict__ gout, const BwdArgs a) {
    const int blk = blockIdx.x, b = blockIdx.y;
    const int r0 = blk * kDuRows;
    const int chunks = a.Hq * (kHeadDim / 8);
    for (int c = threadIdx.x; c < chunks; c += blockDim.x) {
        const int h = c / (kHeadDim / 8), d0 = (c % (kHeadDim / 8)) * 8;
        float s[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        const float *gtp = a.coef + ((static_cast<size_t>(b) * a.Hq + h) * a.Tpad + r0) * kBwdCoefWords + kBcGT;
        const __nv_bfloat16 *gp = gout + ((static_cast<size_t>(b) * a.T + r0) * a.Hq + h) * kHeadDim + d0;
        const size_t rstride = static_cast<size_t>(a.Hq) * kHeadDim;
#pragma unroll
        for (int r = 0; r < kDuRows; ++r) {
            if (r0 + r >= a.T) break;
            const float gt = gtp[static_cast<size_t>(r) * kBwdCoefWords];
            const uint4 g = *reinterpret_cast<const uint4 *>(gp + r * rstride);
            const uint32_t gw[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                s[2 * x] = fmaf(gt, __uint_as_float(gw[x] << 16), s[2 * x]);
                s[2 * x + 1] = fmaf(gt, __uint_as_float(gw[x] & 0xFFFF0000u), s[2 * x + 1]);
            }
        }
        float4 *dst = reinterpret_cast<float4 *>(
            a.du_part + ((static_cast<size_t>(b) * gridDim.x + blk) * a.Hq + h) * kHeadDim + d0);
        dst[0] = make_float4(s[0], s[1], s[2], s[3]);
        dst[1] = make_float4(s[4], s[5], s[6], s[7]);
    }
}

// Rows kernel of the backward from a training forward's saved state (bf16):
// per (row, head), the coefficient record and dA from the row's saved
// streaming state, out and g = dL/dout, without the forward sweep.  With
// count = gate * T from the state, content = out - count * u_h (out rounded to
// bf16, as the forward stored it), <content, g> = <out, g> - count <g, u_h>
// and dA = (g - content <content, g>) / |acc|.
// A block takes 16 rows of one batch and up to 8 heads (blockIdx.z: head
// group), in three phases:
//  A. eight threads per (row, head), each with 8 of the 64 components, load
//     g and out (all of a thread's rows at once) and reduce <out, g> and
//     <g, u_h> among themselves;
//  B. one thread per (row, head) turns the saved state into the magnitude
//     channel's scalars and writes the record;
//  C. the eight threads write dA and sum count * g into the du partials (the
//     16-row blocks of bwd_du_part_kernel).
// Rows T .. Tpad - 1 get the null record and dA = 0.
constexpr int kStHeads = 8;                           // heads per block
constexpr int kStChunks = kStHeads * (kHeadDim / 8);  // 64 (head, 8-component) chunks
constexpr int kStGroups = 256 / kStChunks;            // 4 row groups of 64 threads
constexpr int kStRowsPerThread = kDuRows / kStGroups; // rows rg, rg + 4, rg + 8, rg + 12
__global__ void __launch_bounds__(256, 2)
bwd_state_rows_kernel(const __nv_bfloat16 *__restrict__ out, const __nv_bfloat16 *__restrict__ gout,
                      const float *__restrict__ state, const BwdArgs a) {
    __shared__ float s_og[kDuRows][kStHeads], s_gu[kDuRows][kStHeads];
    __shared__ float s_gt[kDuRows][kStHeads], s_cg[kDuRows][kStHeads], s_ia[kDuRows][kStHeads];
    __shared__ __align__(16) float s_du[kStGroups - 1][kStChunks][8];
    const int blk = blockIdx.x, b = blockIdx.y, h0 = blockIdx.z * kStHeads;
    const int nh = min(kStHeads, a.Hq - h0);
    const int r0 = blk * kDuRows;
    const int t = threadIdx.x, c = t % kStChunks, rg = t / kStChunks;
    const int hl = c >> 3, h = h0 + hl, d0 = (c & 7) * 8;
    const bool act = hl < nh;
    const size_t rstride = static_cast<size_t>(a.Hq) * kHeadDim;
    float uu[8];
    {
        const float *up = a.u + static_cast<size_t>(act ? h : h0) * kHeadDim + d0;
        const float4 u0 = *reinterpret_cast<const float4 *>(up);
        const float4 u1 = *reinterpret_cast<const float4 *>(up + 4);
        uu[0] = u0.x; uu[1] = u0.y; uu[2] = u0.z; uu[3] = u0.w;
        uu[4] = u1.x; uu[5] = u1.y; uu[6] = u1.z; uu[7] = u1.w;
    }
    // The saved state of this thread's (row, head) of phase B, loaded with
    // phase A's loads.
    const int brl = t / kStHeads, bhb = t % kStHeads, brow = r0 + brl, bh = h0 + bhb;
    const bool bact = t < kDuRows * kStHeads && bhb < nh && brow < a.Tpad;
    float4 st0 = make_float4(0.f, 0.f, 0.f, 0.f), st1 = st0;
    if (bact && brow < a.T) {
        const float4 *sp = reinterpret_cast<const float4 *>(
            state + ((static_cast<size_t>(b) * a.Hq + bh) * a.T + brow) * kFwdStateWords);
        st0 = sp[0];
        st1 = sp[1];
    }
    // A: every load first, then the 8-lane reductions.
    uint4 gw[kStRowsPerThread], ow[kStRowsPerThread];
#pragma unroll
    for (int i = 0; i < kStRowsPerThread; ++i) {
        const int row = r0 + rg + kStGroups * i;
        const bool live = act && row < a.T;
        const size_t off = (static_cast<size_t>(b) * a.T + (live ? row : 0)) * rstride +
                           static_cast<size_t>(live ? h : 0) * kHeadDim + d0;
        gw[i] = live ? *reinterpret_cast<const uint4 *>(gout + off) : make_uint4(0u, 0u, 0u, 0u);
        ow[i] = live ? *reinterpret_cast<const uint4 *>(out + off) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int i = 0; i < kStRowsPerThread; ++i) {
        const uint32_t g4[4] = {gw[i].x, gw[i].y, gw[i].z, gw[i].w};
        const uint32_t o4[4] = {ow[i].x, ow[i].y, ow[i].z, ow[i].w};
        float og = 0.f, gu = 0.f;
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            const float g0 = __uint_as_float(g4[x] << 16), g1 = __uint_as_float(g4[x] & 0xFFFF0000u);
            og = fmaf(__uint_as_float(o4[x] << 16), g0, og);
            og = fmaf(__uint_as_float(o4[x] & 0xFFFF0000u), g1, og);
            gu = fmaf(g0, uu[2 * x], gu);
            gu = fmaf(g1, uu[2 * x + 1], gu);
        }
#pragma unroll
        for (int o = 1; o < 8; o <<= 1) {
            og += __shfl_xor_sync(0xffffffffu, og, o);
            gu += __shfl_xor_sync(0xffffffffu, gu, o);
        }
        if ((c & 7) == 0) {
            s_og[rg + kStGroups * i][hl] = og;
            s_gu[rg + kStGroups * i][hl] = gu;
        }
    }
    __syncthreads();
    // B: one (row, head) per thread.
    if (bact) {
        const size_t rrow = (static_cast<size_t>(b) * a.Hq + bh) * a.Tpad + brow;
        float gt = 0.f, cg = 0.f, ia = 0.f;
        if (brow < a.T) {
            const float l = st0.x, l2 = st0.y;
            const float n = static_cast<float>(a.window > 0 ? min(brow + 1, a.window) : brow + 1);
            const float cc = a.s * length_temperature(n, a.alpha, a.L);
            const RowMag m = row_mag(l, l2, st0.z, st0.w, st1.x, cc, n, a.beta, a.inv_ln_L);
            const float gu = s_gu[brl][bhb];
            gt = m.gate * m.Tm;
            cg = s_og[brl][bhb] - gt * gu;  // <content, g>
            ia = 1.0f / st1.y;
            const int lo = a.window > 0 ? max(0, brow - a.window + 1) : 0;
            store_coef_record(a.coef + rrow * kBwdCoefWords, true, m, gu, l, l2, cc, cc * kLog2e, n,
                              a.beta, a.inv_ln_L, __float_as_int(st1.z), lo);
        } else {
            store_coef_record(a.coef + rrow * kBwdCoefWords, false, RowMag{}, 0.f, 0.f, 0.f, 0.f, 0.f,
                              1.f, a.beta, a.inv_ln_L, -1, 0);
        }
        s_gt[brl][bhb] = gt;
        s_cg[brl][bhb] = cg;
        s_ia[brl][bhb] = ia;
    }
    __syncthreads();
    // C: dA and the du partials.
    float du[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int i = 0; i < kStRowsPerThread; ++i) {
        const int rl = rg + kStGroups * i, row = r0 + rl;
        if (!act || row >= a.Tpad) continue;
        const size_t rrow = (static_cast<size_t>(b) * a.Hq + h) * a.Tpad + row;
        uint4 *dst = reinterpret_cast<uint4 *>(a.dab + rrow * kHeadDim + d0);
        if (row >= a.T) {
            *dst = make_uint4(0u, 0u, 0u, 0u);
            continue;
        }
        const float gt = s_gt[rl][hl], cg = s_cg[rl][hl], ia = s_ia[rl][hl];
        const uint32_t g4[4] = {gw[i].x, gw[i].y, gw[i].z, gw[i].w};
        const uint32_t o4[4] = {ow[i].x, ow[i].y, ow[i].z, ow[i].w};
        uint32_t d[4];
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            const float g0 = __uint_as_float(g4[x] << 16), g1 = __uint_as_float(g4[x] & 0xFFFF0000u);
            const float c0v = fmaf(-gt, uu[2 * x], __uint_as_float(o4[x] << 16));
            const float c1v = fmaf(-gt, uu[2 * x + 1], __uint_as_float(o4[x] & 0xFFFF0000u));
            d[x] = pk2((g0 - c0v * cg) * ia, (g1 - c1v * cg) * ia);
            du[2 * x] = fmaf(gt, g0, du[2 * x]);
            du[2 * x + 1] = fmaf(gt, g1, du[2 * x + 1]);
        }
        *dst = make_uint4(d[0], d[1], d[2], d[3]);
    }
    if (rg > 0) {
        *reinterpret_cast<float4 *>(&s_du[rg - 1][c][0]) = make_float4(du[0], du[1], du[2], du[3]);
        *reinterpret_cast<float4 *>(&s_du[rg - 1][c][4]) = make_float4(du[4], du[5], du[6], du[7]);
    }
    __syncthreads();
    if (rg == 0 && act) {
#pragma unroll
        for (int g = 0; g < kStGroups - 1; ++g)
#pragma unroll
            for (int x = 0; x < 8; ++x) du[x] += s_du[g][c][x];
        float4 *dp = reinterpret_cast<float4 *>(
            a.du_part + ((static_cast<size_t>(b) * gridDim.x + blk) * a.Hq + h) * kHeadDim + d0);
        dp[0] = make_float4(du[0], du[1], du[2], du[3]);
        dp[1] = make_float4(du[4], du[5], du[6], du[7]);
    }
}

// du_h = sum over the row blocks of their partial sums: sixteen interleaved
// slices of the partials per head, then the slices, all in a fixed order.
constexpr int kDuSlices = 16;
__global__ void __launch_bounds__(kDuSlices * kHeadDim)
bwd_du_kernel(float *__restrict__ du, const BwdArgs a, int nparts) {
    __shared__ float red[kDuSlices][kHeadDim];
    const int h = blockIdx.x, d = threadIdx.x & (kHeadDim - 1), sl = threadIdx.x >> 6;
    float s = 0.0f;
#pragma unroll 8
    for (int p = sl; p < nparts; p += kDuSlices)
        s += a.du_part[(static_cast<size_t>(p) * a.Hq + h) * kHeadDim + d];
    red[sl][d] = s;
    __syncthreads();
    if (sl == 0) {
        float t = 0.0f;
#pragma unroll
        for (int i = 0; i < kDuSlices; ++i) t += red[i][d];
        du[static_cast<size_t>(h) * kHeadDim + d] = t;
    }
}

template <typename T>
cudaError_t launch_all(const BwdLaunch &l, const BwdArgs &a) {
    const T *q = static_cast<const T *>(l.q), *k = static_cast<const T *>(l.k),
            *v = static_cast<const T *>(l.v), *go = static_cast<const T *>(l.dout);
    int nparts;
    if constexpr (std::is_same<T, __nv_bfloat16>::value) {
        // Rows pass: the forward's tcgen05 sweep where it applies, else the
        // mma.sync kernel (which also writes the du partials).
        int launched = 0;
        cudaError_t e = launch_bwd_rows_tc(l, a.coef, a.dab, a.Tpad);
        if (e == cudaSuccess) {
            nparts = a.B * (a.Tpad / kDuRows);
            bwd_du_part_kernel<<<dim3(a.Tpad / kDuRows, a.B), 128, 0, l.stream>>>(go, a);
            launched = 1;
        } else if (e == cudaErrorNotSupported) {
            nparts = a.B * (a.Tpad / 64);
            bwd_rows_mma_kernel<<<dim3(a.Tpad / 64, a.Hq, a.B), 128, 0, l.stream>>>(q, k, v, go, a);
            launched = 1;
        } else {
            return e;
        }
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        e = launch_bwd_tc(l, a.coef, a.dab);
        if (e != cudaSuccess) return e;
        bwd_du_kernel<<<a.Hq, kDuSlices * kHeadDim, 0, l.stream>>>(l.du, a, nparts);
        count_launches(launched + 1);
        return cudaGetLastError();
    } else {
        nparts = a.B * ((a.T + kRowsB0 - 1) / kRowsB0);
        bwd_rows_kernel<T><<<dim3((a.T + kRowsB0 - 1) / kRowsB0, a.Hq, a.B), kRowsB0, 0, l.stream>>>(
            q, k, v, go, a);
        bwd_dkdv_kernel<T><<<dim3((a.T + kKeyTile - 1) / kKeyTile, a.Hkv, a.B), 128, 0, l.stream>>>(
            q, k, v, l.dk, l.dv, a);
        bwd_dq_kernel<T><<<dim3((a.T + kKeyTile - 1) / kKeyTile, a.Hq, a.B), 128, 0, l.stream>>>(
            q, k, v, l.dq, a);
    }
    bwd_du_kernel<<<a.Hq, kDuSlices * kHeadDim, 0, l.stream>>>(l.du, a, nparts);
    count_launches(4);
    return cudaGetLastError();
}

}  // namespace

// fp32 inputs: the 80-word records and the per-128-row du partials.  bf16
// inputs: the compact records and dA as bf16, both over T rounded up to 128
// rows, and du partials per 16-row block (per 64-row block after the mma.sync
// rows pass).  The workspace holds either layout.
size_t bwd_workspace_bytes(int B, int T, int Hq) {
    const size_t Tpad = (static_cast<size_t>(T) + 127) / 128 * 128;
    const size_t fp32 = static_cast<size_t>(B) * Hq * T * kRecWords * sizeof(float) +
                        static_cast<size_t>(B) * ((T + kRowsB0 - 1) / kRowsB0) * Hq * kHeadDim *
                            sizeof(float);
    const size_t bf16 = static_cast<size_t>(B) * Hq * Tpad * kBwdCoefWords * sizeof(float) +
                        static_cast<size_t>(B) * Hq * Tpad * kHeadDim * sizeof(__nv_bfloat16) +
                        static_cast<size_t>(B) * (Tpad / kDuRows) * Hq * kHeadDim * sizeof(float);
    return fp32 > bf16 ? fp32 : bf16;
}

namespace {

BwdArgs make_args(const BwdLaunch &l) {
    BwdArgs a;
    a.u = l.u;
    a.B = l.B; a.T = l.T; a.Hq = l.Hq; a.Hkv = l.Hkv; a.window = l.window;
    a.Tpad = (l.T + 127) / 128 * 128;
    float *ws = static_cast<float *>(l.workspace);
    if (l.dtype == POLAR_FP32) {
        a.rec = ws;
        a.du_part = a.rec + static_cast<size_t>(l.B) * l.Hq * l.T * kRecWords;
        a.coef = nullptr;
        a.dab = nullptr;
    } else {
        a.rec = nullptr;
        a.coef = ws;
        a.dab = reinterpret_cast<__nv_bfloat16 *>(
            a.coef + static_cast<size_t>(l.B) * l.Hq * a.Tpad * kBwdCoefWords);
        a.du_part = reinterpret_cast<float *>(a.dab + static_cast<size_t>(l.B) * l.Hq * a.Tpad * kHeadDim);
    }
    a.s = l.s; a.alpha = l.alpha; a.L = static_cast<float>(l.L); a.beta = l.beta;
    a.inv_ln_L = 1.0f / logf(static_cast<float>(l.L));
    return a;
}

}  // namespace

cudaError_t launch_bwd(const BwdLaunch &l) {
    const BwdArgs a = make_args(l);
    if (l.B == 0 || l.T == 0) return cudaSuccess;
    return l.dtype == POLAR_FP32 ? launch_all<float>(l, a) : launch_all<__nv_bfloat16>(l, a);
}

// From a training forward's saved state: the state rows kernel (record, dA and
// du partials), the tensor-core dK/dV and dQ passes, du.  Where the training
// forward saved no state (fwd_state_supported false for this shape), the rows
// are recomputed as in launch_bwd.
cudaError_t launch_bwd_from_state(const BwdLaunch &l, const void *out, const float *state) {
    const int sup = fwd_state_supported(l.dtype, l.T, l.Hq, l.Hkv, l.s, l.alpha, l.L, l.window);
    if (sup < 0) return cudaErrorUnknown;
    if (sup == 0) return launch_bwd(l);
    const BwdArgs a = make_args(l);
    if (l.B == 0 || l.T == 0) return cudaSuccess;
    bwd_state_rows_kernel<<<dim3(a.Tpad / kDuRows, a.B, (a.Hq + kStHeads - 1) / kStHeads), 256, 0,
                            l.stream>>>(
        static_cast<const __nv_bfloat16 *>(out), static_cast<const __nv_bfloat16 *>(l.dout), state, a);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    e = launch_bwd_tc(l, a.coef, a.dab);
    if (e != cudaSuccess) return e;
    bwd_du_kernel<<<a.Hq, kDuSlices * kHeadDim, 0, l.stream>>>(l.du, a, a.B * (a.Tpad / kDuRows));
    count_launches(2);
    return cudaGetLastError();
}

}  // namespace polar
