// gdelta.cu -- the recurrent memory channel: a gated-delta associative memory,
// the third additive stream of a Polar Attention layer ("ATMA: Length-
// Invariant Language Modeling via Polar Attention and Gated-Delta Compression
// Memory", gist.science technical summary, section 2.1 "Recurrent Memory
// Channel"; section 2.2 "In-Place Gated-Delta Step Kernel").
//
// Per (sequence, head), state S (64 x 64, row = value dim, column = key dim):
//   S_t = alpha_t S_{t-1} (I - beta_t kh kh^T) + beta_t v_t kh^T,  o_t = S_t qh
// with qh, kh the L2-normalised query and key (the stability mechanism).
//
// Prefill runs chunk-parallel (64 tokens a chunk).  Inside a chunk, with
// g_t = sum_{s<=t} ln alpha_s (chunk-local, inclusive) and b_t = exp(g_t), the
// rank-one writes u_t = S_t - alpha_t S_{t-1} applied to kh_t satisfy
//   u_t + beta_t sum_{j<t} e^{g_t-g_j} <kh_t,kh_j> u_j = beta_t (v_t - b_t S_0 kh_t),
// a unit lower-triangular system (I + A) U = diag(beta) V - diag(beta b) Kh S_0^T.
// Writing W = (I+A)^-1 diag(beta b) Kh and Ut = (I+A)^-1 diag(beta) V (both
// independent of S_0):
//   U   = Ut - W S_0^T
//   O   = diag(b) Qh S_0^T + (e^{g_t-g_j} <qh_t,kh_j>)_{j<=t} U
//   S_C = b_last S_0 + U^T diag(e^{g_last-g_j}) Kh
// Kernel 1 (one CTA per chunk, all chunks in parallel) forms A, the masked
// query-key matrix P, solves for W and Ut, and stores them with the row scales.
// Kernel 2 (one CTA per (sequence, head, 16 value rows); state rows evolve
// independently) walks the chunks in order and applies the three products to
// its slice of the state.  All arithmetic is fp32 on the CUDA cores.
//
// The decode step updates S in place in its pool slot: one read and one write
// of the 16 KB state per (sequence, head), the rank-one form of the update.
#include "polar_common.cuh"
#include "polar_gdelta.h"
#include "polar_internal.h"

namespace polar {
namespace {

constexpr int kC = 64;                 // tokens per chunk
constexpr int kPitch = 68;             // fp32 row pitch in shared memory (272 B)
constexpr int kSlice = 16;             // value rows of the state per scan CTA
constexpr int kWsFloats = 3 * 4096 + 192;  // W, Ut, P, then qs[64], ks[64], b_last
constexpr int kWsQs = 3 * 4096, kWsKs = kWsQs + 64, kWsBlast = kWsKs + 64;
constexpr float kMinLogAlpha = -87.0f;  // alpha below e^-87 (1.6e-38) acts as e^-87

template <typename Tin>
__device__ __forceinline__ float to_f(Tin x);
template <>
__device__ __forceinline__ float to_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename Tin>
__device__ __forceinline__ Tin from_f(float x);
template <>
__device__ __forceinline__ float from_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16(x); }

// Rows [0, n) of one (sequence, head) chunk of a [B, T, H, 64] tensor into a
// [64][kPitch] fp32 shared tile, rows >= n zero.  `rowscale` (shared, or null)
// multiplies each row.  256 threads.
template <typename Tin>
__device__ __forceinline__ void load_rows(float *dst, const Tin *src, size_t row0, int H, int n,
                                          const float *rowscale) {
    constexpr int kPer = 16 / sizeof(Tin);          // elements per 16-byte piece
    constexpr int kPieces = kC * (64 / kPer);       // pieces in the tile
    for (int p = threadIdx.x; p < kPieces; p += blockDim.x) {
        const int t = p / (64 / kPer), c0 = (p % (64 / kPer)) * kPer;
        float vals[kPer];
        if (t < n) {
            const uint4 raw = *reinterpret_cast<const uint4 *>(
                src + ((row0 + t) * H) * static_cast<size_t>(kHeadDim) + c0);
            const Tin *e = reinterpret_cast<const Tin *>(&raw);
            const float sc = rowscale ? rowscale[t] : 1.0f;
#pragma unroll
            for (int i = 0; i < kPer; ++i) vals[i] = to_f<Tin>(e[i]) * sc;
        } else {
#pragma unroll
            for (int i = 0; i < kPer; ++i) vals[i] = 0.0f;
        }
#pragma unroll
        for (int i = 0; i < kPer; i += 4)
            *reinterpret_cast<float4 *>(dst + t * kPitch + c0 + i) =
                make_float4(vals[i], vals[i + 1], vals[i + 2], vals[i + 3]);
    }
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

__device__ __forceinline__ float dot4(float4 a, float4 b, float acc) {
    acc = fmaf(a.x, b.x, acc);
    acc = fmaf(a.y, b.y, acc);
    acc = fmaf(a.z, b.z, acc);
    return fmaf(a.w, b.w, acc);
}

// Normalises rows [8w, 8w + 8) of a [64][kPitch] tile in place (warp w of 8)
// and stores 1/|row| (0 for a zero row) in inv[].
__device__ __forceinline__ void normalise_rows(float *tile, float *inv) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int t = 8 * warp + i;
        float a = tile[t * kPitch + lane], b = tile[t * kPitch + lane + 32];
        const float ss = warp_sum(fmaf(a, a, b * b));
        const float r = ss > 0.0f ? 1.0f / sqrtf(ss) : 0.0f;
        tile[t * kPitch + lane] = a * r;
        tile[t * kPitch + lane + 32] = b * r;
        if (lane == 0) inv[t] = r;
    }
}

struct GdArgs {
    const void *q, *k, *v;
    const float *alpha, *beta;
    float *state;
    void *out;
    float *ws;
    int B, T, H, nchunks, zero_init, accumulate;
};

// Kernel 1: one CTA per (chunk, sequence x head).
template <typename Tin>
__global__ void __launch_bounds__(256) gd_chunk_kernel(GdArgs a) {
    extern __shared__ __align__(16) float sm[];
    float *Qs = sm, *Ks = Qs + kC * kPitch, *Vs = Ks + kC * kPitch, *As = Vs + kC * kPitch;
    float *gam = As + kC * kPitch, *bet = gam + kC, *rho = bet + kC, *kap = rho + kC,
          *bb = kap + kC;

    const int ch = blockIdx.x, bh = blockIdx.y;
    const int b = bh / a.H, h = bh % a.H;
    const int t0 = ch * kC, n = min(kC, a.T - t0);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const size_t row0 = static_cast<size_t>(b) * a.T + t0;
    float *ws = a.ws + (static_cast<size_t>(bh) * a.nchunks + ch) * kWsFloats;

    load_rows<Tin>(Qs, static_cast<const Tin *>(a.q) + h * kHeadDim, row0, a.H, n, nullptr);
    load_rows<Tin>(Ks, static_cast<const Tin *>(a.k) + h * kHeadDim, row0, a.H, n, nullptr);
    load_rows<Tin>(Vs, static_cast<const Tin *>(a.v) + h * kHeadDim, row0, a.H, n, nullptr);
    if (warp == 0) {
        // inclusive scan of the clamped log gates; padded rows: ln alpha = 0, beta = 0
        float la[2], be[2];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int t = 2 * lane + i;
            const size_t idx = (row0 + t) * a.H + h;
            la[i] = t < n ? fmaxf(logf(a.alpha[idx]), kMinLogAlpha) : 0.0f;
            be[i] = t < n ? a.beta[idx] : 0.0f;
        }
        const float pair = la[0] + la[1];
        float incl = pair;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        const float excl = incl - pair;
        gam[2 * lane] = excl + la[0];
        gam[2 * lane + 1] = incl;
        bet[2 * lane] = be[0];
        bet[2 * lane + 1] = be[1];
        bb[2 * lane] = be[0] * expf(excl + la[0]);
        bb[2 * lane + 1] = be[1] * expf(incl);
    }
    __syncthreads();
    normalise_rows(Qs, rho);
    normalise_rows(Ks, kap);
    __syncthreads();

    // Key-key and query-key products, 4 x 4 tiles of the lower triangle.
    {
        const int tr = tid >> 4, tc = tid & 15;
        float gk[4][4], gq[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) gk[i][j] = gq[i][j] = 0.0f;
        if (tc <= tr) {
#pragma unroll 4
            for (int d = 0; d < 64; d += 4) {
                float4 kt[4], qt[4], kj[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    kt[i] = *reinterpret_cast<const float4 *>(Ks + (4 * tr + i) * kPitch + d);
                    qt[i] = *reinterpret_cast<const float4 *>(Qs + (4 * tr + i) * kPitch + d);
                    kj[i] = *reinterpret_cast<const float4 *>(Ks + (4 * tc + i) * kPitch + d);
                }
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        gk[i][j] = dot4(kt[i], kj[j], gk[i][j]);
                        gq[i][j] = dot4(qt[i], kj[j], gq[i][j]);
                    }
            }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int t = 4 * tr + i;
            float av[4], pv[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int jj = 4 * tc + j;
                const float e = jj <= t ? expf(gam[t] - gam[jj]) : 0.0f;
                av[j] = jj < t ? bet[t] * e * gk[i][j] : 0.0f;
                pv[j] = e * gq[i][j];
            }
            *reinterpret_cast<float4 *>(As + t * kPitch + 4 * tc) =
                make_float4(av[0], av[1], av[2], av[3]);
            *reinterpret_cast<float4 *>(ws + 2 * 4096 + t * 64 + 4 * tc) =
                make_float4(pv[0], pv[1], pv[2], pv[3]);
        }
    }
    __syncthreads();

    if (tid < 128) {
        // Forward substitution for one column of [diag(beta b) Kh | diag(beta) V].
        const int c = tid;
        float x[kC];
#pragma unroll
        for (int t = 0; t < kC; ++t)
            x[t] = c < 64 ? bb[t] * Ks[t * kPitch + c] : bet[t] * Vs[t * kPitch + c - 64];
#pragma unroll
        for (int t = 1; t < kC; ++t) {
            float acc = x[t];
#pragma unroll
            for (int g = 0; g < (t + 3) / 4; ++g) {
                const float4 av = *reinterpret_cast<const float4 *>(As + t * kPitch + 4 * g);
                acc = fmaf(-av.x, x[4 * g], acc);
                acc = fmaf(-av.y, x[4 * g + 1], acc);
                acc = fmaf(-av.z, x[4 * g + 2], acc);
                acc = fmaf(-av.w, x[4 * g + 3], acc);
            }
            x[t] = acc;
        }
        float *dst = c < 64 ? ws + c : ws + 4096 + (c - 64);
#pragma unroll
        for (int t = 0; t < kC; ++t) dst[t * 64] = x[t];
    } else if (tid < 192) {
        const int t = tid - 128;
        const float glast = gam[kC - 1];
        ws[kWsQs + t] = rho[t] * expf(gam[t]);
        ws[kWsKs + t] = kap[t] * expf(glast - gam[t]);
        if (t == 0) ws[kWsBlast] = expf(glast);
    }
}

// Kernel 2: one CTA per (16 value rows, sequence x head); walks the chunks.
template <typename Tin>
__global__ void __launch_bounds__(256) gd_scan_kernel(GdArgs a) {
    extern __shared__ __align__(16) float sm[];
    float *Wsm = sm, *Psm = Wsm + kC * kPitch, *Qsm = Psm + kC * kPitch, *Ksm = Qsm + kC * kPitch;
    float *Ssm = Ksm + kC * kPitch, *Ut = Ssm + kSlice * kPitch;
    float *qs = Ut + kSlice * kPitch, *ks = qs + kC;

    const int slice = blockIdx.x, bh = blockIdx.y;
    const int b = bh / a.H, h = bh % a.H;
    const int r0 = slice * kSlice;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    float *state = a.state + (static_cast<size_t>(bh) * 64 + r0) * 64;

    for (int i = tid; i < kSlice * 64; i += 256) {
        const int r = i >> 6, c = i & 63;
        Ssm[r * kPitch + c] = a.zero_init ? 0.0f : state[r * 64 + c];
    }

    // Products over (token t, value row r): r = lane % 16, t = 4 tg + i.
    const int r = lane & 15, tg = 2 * warp + (lane >> 4);
    // State update over (value row rs, key column 4 cq + i).
    const int rs = 2 * warp + (lane >> 4), cq = lane & 15;
    const Tin *qsrc = static_cast<const Tin *>(a.q) + h * kHeadDim;
    const Tin *ksrc = static_cast<const Tin *>(a.k) + h * kHeadDim;
    Tin *out = static_cast<Tin *>(a.out);

    for (int ch = 0; ch < a.nchunks; ++ch) {
        const int t0 = ch * kC, n = min(kC, a.T - t0);
        const size_t row0 = static_cast<size_t>(b) * a.T + t0;
        const float *ws = a.ws + (static_cast<size_t>(bh) * a.nchunks + ch) * kWsFloats;
        if (tid < 64) qs[tid] = ws[kWsQs + tid];
        else if (tid < 128) ks[tid - 64] = ws[kWsKs + tid - 64];
        for (int i = tid; i < 1024; i += 256) {
            const int t = i >> 4, c = (i & 15) * 4;
            *reinterpret_cast<float4 *>(Wsm + t * kPitch + c) =
                *reinterpret_cast<const float4 *>(ws + t * 64 + c);
            *reinterpret_cast<float4 *>(Psm + t * kPitch + c) =
                *reinterpret_cast<const float4 *>(ws + 2 * 4096 + t * 64 + c);
        }
        float u[4], oi[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            u[i] = ws[4096 + (4 * tg + i) * 64 + r0 + r];
            oi[i] = 0.0f;
        }
        const float blast = ws[kWsBlast];
        __syncthreads();  // qs, ks visible; previous chunk's readers of Qsm/Ksm done
        load_rows<Tin>(Qsm, qsrc, row0, a.H, n, qs);
        load_rows<Tin>(Ksm, ksrc, row0, a.H, n, ks);
        __syncthreads();

        // U = Ut - W S^T and the inter-chunk read diag(b) Qh S^T.
#pragma unroll 4
        for (int c = 0; c < 64; c += 4) {
            const float4 s4 = *reinterpret_cast<const float4 *>(Ssm + r * kPitch + c);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float4 w4 = *reinterpret_cast<const float4 *>(Wsm + (4 * tg + i) * kPitch + c);
                const float4 q4 = *reinterpret_cast<const float4 *>(Qsm + (4 * tg + i) * kPitch + c);
                u[i] = dot4(make_float4(-w4.x, -w4.y, -w4.z, -w4.w), s4, u[i]);
                oi[i] = dot4(q4, s4, oi[i]);
            }
        }
        *reinterpret_cast<float4 *>(Ut + r * kPitch + 4 * tg) = make_float4(u[0], u[1], u[2], u[3]);
        __syncthreads();

        // O = inter + P U (P is zero above the diagonal).
        for (int g = 0; g <= tg; ++g) {
            const float4 u4 = *reinterpret_cast<const float4 *>(Ut + r * kPitch + 4 * g);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float4 p4 = *reinterpret_cast<const float4 *>(Psm + (4 * tg + i) * kPitch + 4 * g);
                oi[i] = dot4(p4, u4, oi[i]);
            }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int t = 4 * tg + i;
            if (t < n) {
                Tin *dst = out + ((row0 + t) * a.H + h) * static_cast<size_t>(kHeadDim) + r0 + r;
                const float val = a.accumulate ? to_f<Tin>(*dst) + oi[i] : oi[i];
                *dst = from_f<Tin>(val);
            }
        }

        // S <- b_last S + U^T diag(ks) K (ks folded into Ksm).
        float sn[4];
        {
            const float4 s4 = *reinterpret_cast<const float4 *>(Ssm + rs * kPitch + 4 * cq);
            sn[0] = blast * s4.x; sn[1] = blast * s4.y; sn[2] = blast * s4.z; sn[3] = blast * s4.w;
        }
#pragma unroll 4
        for (int j = 0; j < 64; j += 4) {
            const float4 u4 = *reinterpret_cast<const float4 *>(Ut + rs * kPitch + j);
            const float uj[4] = {u4.x, u4.y, u4.z, u4.w};
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                const float4 k4 = *reinterpret_cast<const float4 *>(Ksm + (j + jj) * kPitch + 4 * cq);
                sn[0] = fmaf(uj[jj], k4.x, sn[0]);
                sn[1] = fmaf(uj[jj], k4.y, sn[1]);
                sn[2] = fmaf(uj[jj], k4.z, sn[2]);
                sn[3] = fmaf(uj[jj], k4.w, sn[3]);
            }
        }
        __syncthreads();  // every read of Ssm and Ut in this chunk is done
        *reinterpret_cast<float4 *>(Ssm + rs * kPitch + 4 * cq) = make_float4(sn[0], sn[1], sn[2], sn[3]);
    }
    __syncthreads();
    for (int i = tid; i < kSlice * 64; i += 256) {
        const int rr = i >> 6, c = i & 63;
        state[rr * 64 + c] = Ssm[rr * kPitch + c];
    }
}

// Decode step: one CTA per (sequence, head); thread owns S[tid/4][16 (tid%4) .. +16).
template <typename Tin>
__global__ void __launch_bounds__(256) gd_step_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k,
                                                      const Tin *__restrict__ v,
                                                      const float *__restrict__ alpha,
                                                      const float *__restrict__ beta, float *pool,
                                                      int num_slots, const int32_t *__restrict__ slots,
                                                      int H, Tin *out, int accumulate, int *status) {
    __shared__ float qh[64], kh[64], vv[64];
    const int seq = blockIdx.x / H, h = blockIdx.x % H;
    const int slot = slots[seq];
    if (slot < 0) return;
    if (slot >= num_slots) {
        if (threadIdx.x == 0) record_error(status, POLAR_ERR_BAD_SLOT);
        return;
    }
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int r = tid >> 2, c0 = 16 * (tid & 3);
    float *S = pool + ((static_cast<size_t>(slot) * H + h) * 64 + r) * 64 + c0;
    float4 s[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) s[i] = reinterpret_cast<const float4 *>(S)[i];
    const size_t row = static_cast<size_t>(seq) * H + h;
    if (warp < 3) {
        const Tin *src = (warp == 0 ? q : warp == 1 ? k : v) + row * kHeadDim;
        float x0 = to_f<Tin>(src[lane]), x1 = to_f<Tin>(src[lane + 32]);
        if (warp < 2) {
            const float ss = warp_sum(fmaf(x0, x0, x1 * x1));
            const float inv = ss > 0.0f ? 1.0f / sqrtf(ss) : 0.0f;
            x0 *= inv;
            x1 *= inv;
        }
        float *dst = warp == 0 ? qh : warp == 1 ? kh : vv;
        dst[lane] = x0;
        dst[lane + 32] = x1;
    }
    const float al = alpha[row], be = beta[row];
    __syncthreads();

    float sk = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float4 k4 = *reinterpret_cast<const float4 *>(kh + c0 + 4 * i);
        sk = dot4(s[i], k4, sk);
    }
    sk += __shfl_xor_sync(0xffffffffu, sk, 1);
    sk += __shfl_xor_sync(0xffffffffu, sk, 2);
    const float w = be * (vv[r] - al * sk);
    float o = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float4 k4 = *reinterpret_cast<const float4 *>(kh + c0 + 4 * i);
        const float4 q4 = *reinterpret_cast<const float4 *>(qh + c0 + 4 * i);
        s[i].x = fmaf(al, s[i].x, w * k4.x);
        s[i].y = fmaf(al, s[i].y, w * k4.y);
        s[i].z = fmaf(al, s[i].z, w * k4.z);
        s[i].w = fmaf(al, s[i].w, w * k4.w);
        o = dot4(s[i], q4, o);
        reinterpret_cast<float4 *>(S)[i] = s[i];
    }
    o += __shfl_xor_sync(0xffffffffu, o, 1);
    o += __shfl_xor_sync(0xffffffffu, o, 2);
    if ((tid & 3) == 0) {
        Tin *dst = out + row * kHeadDim + r;
        *dst = from_f<Tin>(accumulate ? to_f<Tin>(*dst) + o : o);
    }
}

constexpr size_t kChunkSmem = (4 * kC * kPitch + 5 * kC) * sizeof(float);
constexpr size_t kScanSmem = (4 * kC * kPitch + 2 * kSlice * kPitch + 2 * kC) * sizeof(float);

template <typename Tin>
cudaError_t launch_prefill_t(const GdArgs &g, cudaStream_t stream) {
    static bool configured = false;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(gd_chunk_kernel<Tin>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(kChunkSmem));
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(gd_scan_kernel<Tin>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(kScanSmem));
        if (e != cudaSuccess) return e;
        configured = true;
    }
    const unsigned bh = static_cast<unsigned>(g.B * g.H);
    gd_chunk_kernel<Tin><<<dim3(g.nchunks, bh), 256, kChunkSmem, stream>>>(g);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    gd_scan_kernel<Tin><<<dim3(64 / kSlice, bh), 256, kScanSmem, stream>>>(g);
    count_launches(2);
    return cudaGetLastError();
}

}  // namespace

size_t gdelta_workspace_bytes(int B, int T, int H) {
    const size_t nch = (static_cast<size_t>(T) + kC - 1) / kC;
    return static_cast<size_t>(B) * H * nch * kWsFloats * sizeof(float);
}

cudaError_t launch_gdelta_prefill(const GdeltaLaunch &l) {
    if (l.B == 0 || l.T == 0) return cudaSuccess;
    GdArgs g;
    g.q = l.q; g.k = l.k; g.v = l.v; g.alpha = l.alpha; g.beta = l.beta;
    g.state = l.state; g.out = l.out; g.ws = static_cast<float *>(l.workspace);
    g.B = l.B; g.T = l.T; g.H = l.H; g.nchunks = (l.T + kC - 1) / kC;
    g.zero_init = l.zero_init; g.accumulate = l.accumulate;
    return l.dtype == POLAR_FP32 ? launch_prefill_t<float>(g, l.stream)
                                 : launch_prefill_t<__nv_bfloat16>(g, l.stream);
}

cudaError_t launch_gdelta_step(const GdeltaStepLaunch &l) {
    if (l.num_seqs == 0) return cudaSuccess;
    const unsigned grid = static_cast<unsigned>(l.num_seqs) * static_cast<unsigned>(l.H);
    if (l.dtype == POLAR_FP32) {
        gd_step_kernel<float><<<grid, 256, 0, l.stream>>>(
            static_cast<const float *>(l.q), static_cast<const float *>(l.k),
            static_cast<const float *>(l.v), l.alpha, l.beta, l.pool, l.num_slots, l.slots, l.H,
            static_cast<float *>(l.out), l.accumulate, l.status);
    } else {
        gd_step_kernel<__nv_bfloat16><<<grid, 256, 0, l.stream>>>(
            static_cast<const __nv_bfloat16 *>(l.q), static_cast<const __nv_bfloat16 *>(l.k),
            static_cast<const __nv_bfloat16 *>(l.v), l.alpha, l.beta, l.pool, l.num_slots,
            l.slots, l.H, static_cast<__nv_bfloat16 *>(l.out), l.accumulate, l.status);
    }
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace polar
