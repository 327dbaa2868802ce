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
// Four launches, all FP32 on the CUDA cores:
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
    float *rec;
    float *du_part;  // [B * row blocks][Hq][64]: per-block sums of gate * T * g
    int B, T, Hq, Hkv, window;
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
    *reinterpret_cast<float4 *>(rec + 72) =
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

// -------------------------------------------------------------------- du ---
// du_h = sum over the row blocks of their partial sums (fixed order).
__global__ void __launch_bounds__(kHeadDim)
bwd_du_kernel(float *__restrict__ du, const BwdArgs a, int nparts) {
    const int h = blockIdx.x, d = threadIdx.x;
    float s = 0.0f;
    for (int p = 0; p < nparts; ++p) s += a.du_part[(static_cast<size_t>(p) * a.Hq + h) * kHeadDim + d];
    du[static_cast<size_t>(h) * kHeadDim + d] = s;
}

template <typename T>
cudaError_t launch_all(const BwdLaunch &l, const BwdArgs &a) {
    const T *q = static_cast<const T *>(l.q), *k = static_cast<const T *>(l.k),
            *v = static_cast<const T *>(l.v), *go = static_cast<const T *>(l.dout);
    bwd_rows_kernel<T><<<dim3((a.T + kRowsB0 - 1) / kRowsB0, a.Hq, a.B), kRowsB0, 0, l.stream>>>(
        q, k, v, go, a);
    bwd_dkdv_kernel<T><<<dim3((a.T + kKeyTile - 1) / kKeyTile, a.Hkv, a.B), 128, 0, l.stream>>>(
        q, k, v, l.dk, l.dv, a);
    bwd_dq_kernel<T><<<dim3((a.T + kKeyTile - 1) / kKeyTile, a.Hq, a.B), 128, 0, l.stream>>>(
        q, k, v, l.dq, a);
    bwd_du_kernel<<<a.Hq, kHeadDim, 0, l.stream>>>(l.du, a, a.B * ((a.T + kRowsB0 - 1) / kRowsB0));
    count_launches(4);
    return cudaGetLastError();
}

}  // namespace

size_t bwd_workspace_bytes(int B, int T, int Hq) {
    const size_t rec = static_cast<size_t>(B) * Hq * T * kRecWords * sizeof(float);
    const size_t part =
        static_cast<size_t>(B) * ((T + kRowsB0 - 1) / kRowsB0) * Hq * kHeadDim * sizeof(float);
    return rec + part;
}

cudaError_t launch_bwd(const BwdLaunch &l) {
    BwdArgs a;
    a.u = l.u;
    a.rec = static_cast<float *>(l.workspace);
    a.du_part = a.rec + static_cast<size_t>(l.B) * l.Hq * l.T * kRecWords;
    a.B = l.B; a.T = l.T; a.Hq = l.Hq; a.Hkv = l.Hkv; a.window = l.window;
    a.s = l.s; a.alpha = l.alpha; a.L = static_cast<float>(l.L); a.beta = l.beta;
    a.inv_ln_L = 1.0f / logf(static_cast<float>(l.L));
    if (l.B == 0 || l.T == 0) return cudaSuccess;
    return l.dtype == POLAR_FP32 ? launch_all<float>(l, a) : launch_all<__nv_bfloat16>(l, a);
}

}  // namespace polar
