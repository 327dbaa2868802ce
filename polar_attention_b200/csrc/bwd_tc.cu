// bwd_tc.cu -- tcgen05/TMEM tensor-core passes of the causal Polar Attention
// prefill backward for bf16 inputs (the training use of the fused step of
// "Fused Polar Attention Kernel", ATMA technical summary, section 2.2; the
// chain rule through the three channels of section 2.1).
//
// After the rows pass has written, per query row i, the coefficients of
//   w_ij  = 2^(cl2_i S_ij + nref_i)                     (the row's weights)
//   dS_ij = w_ij (c_i <dA_i, v_j> + e1_i + e2_i w_ij) + e3_i S_ij + e4_i
//           (+ c_i dm_i at the row's first argmax)
// and dA_i rounded to bf16, the gradients are tile products:
//   dV = W^T dA,   dK = dS^T Q,   dQ = dS K.
// Both passes below recompute S = Q K^T and <dA, v> = dA V^T on the tensor
// cores into tensor memory, with the query rows as the 128 TMEM lanes, so each
// coefficient thread owns one row and keeps that row's coefficients in
// registers.
//
// dK/dV pass: one CTA per (128-key tile, kv head, batch).  Q, dA and the rows'
// coefficient records stream through a three-stage ring for every query tile at
// or after the key tile and every query head of the group.  The coefficient
// threads write W and dS as one bf16 tile each in shared memory, row by row
// (a row's 128 keys contiguous, 128B-swizzled), which the tensor core reads as
// the MN-major A operands W^T and dS^T of dV += W^T dA and dK += dS^T Q; dK and
// dV accumulate in tensor memory (keys as lanes) over the whole loop.
//
// dQ pass: one CTA per (128-row query tile, query head, batch), the forward's
// layout: K and V tiles stream through a four-stage ring; dS goes to tensor
// memory as bf16 (two buffers, so that the coefficient threads never wait for
// the previous tile's dQ product) and is the A operand of dQ += dS K.  The argmax term
// c dm k_{jmax} is added in fp32 in the epilogue.
//
// Warp roles (384 threads): warp 0 the TMA producer, warp 1 the tensor-memory
// allocator and single-thread MMA issuer, warps 2-3 idle, warps 4-11 two
// coefficient warpgroups (keys 0-63 and 64-127 of every tile).  Every wait is
// bounded (mbar_wait): on a timeout the kernel records POLAR_ERR_TIMEOUT and
// leaves its loop.
#include <atomic>
#include <mutex>

#include "polar_common.cuh"
#include "polar_internal.h"
#include "tc_common.cuh"

namespace polar {
namespace {

constexpr int kTl = 128;                       // rows per query tile = keys per key tile
constexpr int kTileB = kTl * 128;              // bytes of a 128 x 64 bf16 tile
constexpr int kCoefTileB = kTl * kBwdCoefWords * 4;  // 8 KB

// dK/dV pass shared memory: K, V | 3 stages x (Q, dA, coefficients) | W, dS
// (217 KB).
constexpr int kKvStages = 3;
constexpr int kKvStageB = 2 * kTileB + kCoefTileB;
constexpr int kDkdvSmem = 2 * kTileB + kKvStages * kKvStageB + 4 * kTileB + 1024;
// dQ pass shared memory: Q, dA | 4 stages x (K, V) (161 KB).
constexpr int kDqStages = 4;
constexpr int kDqSmem = 2 * kTileB + kDqStages * 2 * kTileB + 1024;

// Tensor-memory columns (512 allocated).  Both passes: S 0-127, <dA, v> 128-255.
constexpr uint32_t kColS = 0, kColAV = 128;
constexpr uint32_t kColDK = 256, kColDV = 320;  // dK/dV pass (fp32, keys as lanes)
constexpr uint32_t kColDS = 256, kColDQ = 384;  // dQ pass: dS (bf16 pairs, two buffers), dQ (fp32)

struct BwdTcArgs {
    const float *coef;            // [B][Hq][Tpad][kBwdCoefWords]
    const __nv_bfloat16 *k;       // [B][T][Hkv][64] (dQ epilogue: the argmax key)
    float *dq, *dk, *dv;
    int *status;
    int B, T, Tpad, Hq, Hkv, G, nt, window;
};

__device__ __forceinline__ uint8_t *align1024(uint8_t *p) {
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// dS (and, for the dK/dV pass, w) for 64 keys of one row, two at a time:
// keys e, e+1 of the half are visible iff e_lo <= e <= e_hi (kMask only).
template <bool kMask, bool kWantW>
__device__ __forceinline__ void pair_grads(const uint32_t (&s)[2][32], const uint32_t (&av)[2][32],
                                           float4 c0, float4 c1, int e_lo, int e_hi,
                                           uint32_t (&wp)[32], uint32_t (&dp)[32]) {
    const float2 cl2 = make_float2(c0.x, c0.x), nref = make_float2(c0.y, c0.y);
    const float2 cc = make_float2(c0.z, c0.z), e1 = make_float2(c0.w, c0.w);
    const float2 e2 = make_float2(c1.x, c1.x), e3 = make_float2(c1.y, c1.y);
    const float2 e4 = make_float2(c1.z, c1.z);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const float2 sv = make_float2(__uint_as_float(s[h][2 * e]), __uint_as_float(s[h][2 * e + 1]));
            const float2 avv = make_float2(__uint_as_float(av[h][2 * e]), __uint_as_float(av[h][2 * e + 1]));
            const float2 x = f2_fma(sv, cl2, nref);
            float2 w = make_float2(ex2(x.x), ex2(x.y));
            float2 t = f2_fma(avv, cc, e1);
            t = f2_fma(w, e2, t);
            const float2 t2 = f2_fma(sv, e3, e4);
            float2 ds = f2_fma(w, t, t2);
            if (kMask) {
                const int col = 32 * h + 2 * e;
                const bool v0 = col >= e_lo && col <= e_hi, v1 = col + 1 >= e_lo && col + 1 <= e_hi;
                w.x = v0 ? w.x : 0.f;
                w.y = v1 ? w.y : 0.f;
                ds.x = v0 ? ds.x : 0.f;
                ds.y = v1 ? ds.y : 0.f;
            }
            if (kWantW) wp[16 * h + e] = pack_bf16(w.x, w.y);
            dp[16 * h + e] = pack_bf16(ds.x, ds.y);
        }
    }
}

// ------------------------------------------------------------ dK, dV pass ---
__global__ void __launch_bounds__(384, 1)
bwd_dkdv_tc_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                   const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tda,
                   const BwdTcArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024(smem_raw);
    uint8_t *sK = smem, *sV = smem + kTileB;
    uint8_t *sStage = smem + 2 * kTileB;                      // stage s: Q, dA, coefficients
    uint8_t *sW = sStage + kKvStages * kKvStageB;             // W: 2 key blocks x 128 rows x 128 B
    uint8_t *sD = sW + 2 * kTileB;                            // dS, same layout

    __shared__ __align__(8) uint64_t kv_full, st_full, st_free, wd_full, wd_free, acc_done, mma_idle;
    __shared__ __align__(8) uint64_t stage_full[kKvStages], stage_empty[kKvStages];
    __shared__ uint32_t tmem_base_sh;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int per_kt = a.Hkv * a.B;
    const int kt = static_cast<int>(blockIdx.x) / per_kt;   // longest key tiles first
    const int rem = static_cast<int>(blockIdx.x) % per_kt;
    const int g = rem % a.Hkv, b = rem / a.Hkv;
    const int key0 = kt * kTl;
    // Query tiles whose rows see a key of this tile: kt .. qt_hi.
    const int qt_hi = a.window > 0 ? min(a.nt - 1, (key0 + kTl - 1 + a.window - 1) / kTl) : a.nt - 1;
    const int nq = qt_hi - kt + 1;
    const int niter = a.G * nq;  // iteration n: head g*G + n/nq, query tile kt + n%nq

    if (warp == 0 && lane == 0) {
        mbar_init(&kv_full, 1);
        mbar_init(&st_full, 1);
        mbar_init(&st_free, 8);   // one arrival per coefficient warp
        mbar_init(&wd_full, 8);
        mbar_init(&wd_free, 1);
        mbar_init(&acc_done, 1);
        mbar_init(&mma_idle, 1);
        for (int s = 0; s < kKvStages; ++s) {
            mbar_init(&stage_full[s], 1);
            mbar_init(&stage_empty[s], 1);
        }
        fence_barrier_init();
    }
    if (warp == 1) tmem_alloc_512(&tmem_base_sh);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_sh;

    if (warp < 4) {
        reg_dealloc<64>();
        if (warp == 0 && lane == 0) {
            // --------------------------------------------------- TMA producer
            tma_prefetch_desc(&tq);
            tma_prefetch_desc(&tk);
            tma_prefetch_desc(&tv);
            tma_prefetch_desc(&tda);
            mbar_arrive_expect_tx(&kv_full, 2 * kTileB);
            tma_load_4d(sK, &tk, 0, g, key0, b, &kv_full);
            tma_load_4d(sV, &tv, 0, g, key0, b, &kv_full);
            int issued = 0;
            bool ok = true;
            for (int n = 0; n < niter && ok; ++n) {
                const int s = n % kKvStages;
                if (n >= kKvStages &&
                    !(ok = mbar_wait(&stage_empty[s], ((n / kKvStages) - 1) & 1, a.status)))
                    break;
                const int h = g * a.G + n / nq, qt = kt + n % nq;
                uint8_t *st = sStage + s * kKvStageB;
                mbar_arrive_expect_tx(&stage_full[s], 2 * kTileB + kCoefTileB);
                tma_load_4d(st, &tq, 0, h, qt * kTl, b, &stage_full[s]);
                tma_load_3d(st + kTileB, &tda, 0, qt * kTl, b * a.Hq + h, &stage_full[s]);
                bulk_load(st + 2 * kTileB,
                          a.coef + ((static_cast<size_t>(b) * a.Hq + h) * a.Tpad + qt * kTl) * kBwdCoefWords,
                          kCoefTileB, &stage_full[s]);
                ++issued;
            }
            // Every copy this thread started lands before shared memory is released.
            mbar_wait(&kv_full, 0, a.status);
            for (int n = (issued > kKvStages ? issued - kKvStages : 0); n < issued; ++n)
                mbar_wait(&stage_full[n % kKvStages], (n / kKvStages) & 1, a.status);
        } else if (warp == 1 && lane == 0) {
            // ---------------------------------------------------- MMA issuer
            constexpr uint32_t idesc_s = idesc_bf16(kTl, kTl, false);           // Q K^T, dA V^T
            constexpr uint32_t idesc_acc = idesc_bf16(kTl, 64, true, true);     // W^T dA, dS^T Q
            const uint32_t hi = kSdescHi128B;
            const uint32_t k_lo = sdesc_lo(smem_u32(sK), 16), v_lo = sdesc_lo(smem_u32(sV), 16);
            // W^T and dS^T: MN-major A operands whose two 64-key blocks are kTileB apart.
            const uint32_t w_lo = sdesc_lo(smem_u32(sW), kTileB);
            const uint32_t d_lo = sdesc_lo(smem_u32(sD), kTileB);
            bool ok = mbar_wait(&kv_full, 0, a.status);
            auto stage_lo = [&](int s, int which, uint32_t lbo) {
                return sdesc_lo(smem_u32(sStage + s * kKvStageB + which * kTileB), lbo);
            };
            // dV += W^T dA, dK += dS^T Q for iteration m (stage m % 2).
            auto issue_acc = [&](int m) {
                if (!(ok = ok && mbar_wait(&wd_full, m & 1, a.status))) return;
                tc_fence_after();
                const int s = m % kKvStages;
                const uint32_t q_mn = stage_lo(s, 0, 8192), da_mn = stage_lo(s, 1, 8192);
#pragma unroll
                for (int kk = 0; kk < kTl / 16; ++kk)
                    mma_ss_rt(tmem + kColDV, w_lo + 128 * kk, hi, da_mn + 128 * kk, hi, idesc_acc,
                              (m > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
                for (int kk = 0; kk < kTl / 16; ++kk)
                    mma_ss_rt(tmem + kColDK, d_lo + 128 * kk, hi, q_mn + 128 * kk, hi, idesc_acc,
                              (m > 0 || kk > 0) ? 1u : 0u);
                tc_commit(&wd_free);
                tc_commit(&stage_empty[s]);
            };
            for (int n = 0; n < niter && ok; ++n) {
                const int s = n % kKvStages;
                if (!(ok = mbar_wait(&stage_full[s], (n / kKvStages) & 1, a.status))) break;
                if (n > 0 && !(ok = mbar_wait(&st_free, (n - 1) & 1, a.status))) break;
                tc_fence_after();
                const uint32_t q_k = stage_lo(s, 0, 16), da_k = stage_lo(s, 1, 16);
                mma_ss2<0>(tmem + kColS, q_k, hi, k_lo, hi, idesc_s);
#pragma unroll
                for (int kk = 1; kk < 4; ++kk)
                    mma_ss2<1>(tmem + kColS, q_k + 2 * kk, hi, k_lo + 2 * kk, hi, idesc_s);
                mma_ss2<0>(tmem + kColAV, da_k, hi, v_lo, hi, idesc_s);
#pragma unroll
                for (int kk = 1; kk < 4; ++kk)
                    mma_ss2<1>(tmem + kColAV, da_k + 2 * kk, hi, v_lo + 2 * kk, hi, idesc_s);
                tc_commit(&st_full);
                if (n > 0) issue_acc(n - 1);
            }
            if (ok && niter > 0) issue_acc(niter - 1);
            tc_commit(&acc_done);
            // Every MMA this thread issued completes before tensor memory is freed.
            tc_commit(&mma_idle);
            mbar_wait(&mma_idle, 0, a.status);
        }
    } else {
        reg_alloc<208>();
        // ------------------------------------------------- coefficient threads
        const int wg = (warp - 4) >> 2;   // key half: keys 64 wg .. 64 wg + 63 of each tile
        const int wq = warp & 3;          // TMEM lane quarter
        const int t = 32 * wq + lane;     // row within the query tile = TMEM lane
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(32 * wq) << 16);
        const int kbase = key0 + 64 * wg;
        bool ok = true;
        for (int n = 0; n < niter; ++n) {
            const int s = n % kKvStages, qt = kt + n % nq;
            const int i = qt * kTl + t;  // this thread's row
            ok = mbar_wait(&st_full, n & 1, a.status) &&
                 mbar_wait(&stage_full[s], (n / kKvStages) & 1, a.status);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            tc_fence_after();
            const float4 *cr = reinterpret_cast<const float4 *>(sStage + s * kKvStageB + 2 * kTileB +
                                                                t * kBwdCoefWords * 4);
            const float4 c0 = cr[0], c1 = cr[1], c2 = cr[2];
            uint32_t sr[2][32], ar[2][32];
            tmem_ld32(lane_base + kColS + 64 * wg, sr[0]);
            tmem_ld32(lane_base + kColS + 64 * wg + 32, sr[1]);
            tmem_ld32(lane_base + kColAV + 64 * wg, ar[0]);
            tmem_ld32(lane_base + kColAV + 64 * wg + 32, ar[1]);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&st_free);  // the warp's loads are complete
            // Keys of this half visible to row i: lo_i .. i (causal, window).
            const bool masked = qt == kt || (a.window > 0 && qt * kTl + kTl - a.window > key0);
            const int e_hi = i - kbase, e_lo = __float_as_int(c2.y) - kbase;
            uint32_t wp[32], dp[32];
            if (masked)
                pair_grads<true, true>(sr, ar, c0, c1, e_lo, e_hi, wp, dp);
            else
                pair_grads<false, true>(sr, ar, c0, c1, 0, 0, wp, dp);
            // W and dS of the previous iteration consumed: their tiles may be rewritten.
            if (n > 0) {
                ok = mbar_wait(&wd_free, (n - 1) & 1, a.status);
                if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            }
            uint8_t *wrow = sW + wg * kTileB + t * 128;  // key block wg, row t
            uint8_t *drow = sD + wg * kTileB + t * 128;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint32_t off = static_cast<uint32_t>((c ^ (t & 7)) << 4);
                *reinterpret_cast<uint4 *>(wrow + off) =
                    make_uint4(wp[4 * c], wp[4 * c + 1], wp[4 * c + 2], wp[4 * c + 3]);
                *reinterpret_cast<uint4 *>(drow + off) =
                    make_uint4(dp[4 * c], dp[4 * c + 1], dp[4 * c + 2], dp[4 * c + 3]);
            }
            // The max's subgradient: c dm at the row's first argmax, if it is a key of this half.
            const int jm = __float_as_int(c2.x) - kbase;
            if (jm >= 0 && jm < 64) {
                __nv_bfloat16 *p = reinterpret_cast<__nv_bfloat16 *>(
                    drow + ((((jm >> 3) ^ (t & 7))) << 4) + (jm & 7) * 2);
                *p = __float2bfloat16_rn(__bfloat162float(*p) + c1.w);
            }
            fence_proxy_async_smem();  // the tensor core reads W and dS through the async proxy
            __syncwarp();
            if (lane == 0) mbar_arrive(&wd_full);  // after every lane's stores and fence
        }
        // Epilogue: dK (first warpgroup) and dV (second) of key key0 + t.
        if (ok) ok = mbar_wait(&acc_done, 0, a.status);
        if (__all_sync(0xffffffffu, ok) && niter > 0) {
            tc_fence_after();
            uint32_t o[2][32];
            const uint32_t col = wg == 0 ? kColDK : kColDV;
            tmem_ld32(lane_base + col, o[0]);
            tmem_ld32(lane_base + col + 32, o[1]);
            tmem_wait_ld();
            const int j = key0 + t;
            if (j < a.T) {
                float *dst = (wg == 0 ? a.dk : a.dv) +
                             ((static_cast<size_t>(b) * a.T + j) * a.Hkv + g) * kHeadDim;
#pragma unroll
                for (int c = 0; c < 16; ++c)
                    reinterpret_cast<float4 *>(dst)[c] =
                        make_float4(__uint_as_float(o[c >> 3][4 * (c & 7)]),
                                    __uint_as_float(o[c >> 3][4 * (c & 7) + 1]),
                                    __uint_as_float(o[c >> 3][4 * (c & 7) + 2]),
                                    __uint_as_float(o[c >> 3][4 * (c & 7) + 3]));
            }
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

// ------------------------------------------------------------------ dQ pass ---
__global__ void __launch_bounds__(384, 1)
bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                 const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tda,
                 const BwdTcArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024(smem_raw);
    uint8_t *sQ = smem, *sDA = smem + kTileB;
    uint8_t *sKV = smem + 2 * kTileB;  // stage s: K at s * 2 tiles, V after it

    __shared__ __align__(8) uint64_t q_full, st_full, st_free, ds_full, acc_done, mma_idle;
    __shared__ __align__(8) uint64_t ds_free[2], kv_full[kDqStages], kv_empty[kDqStages];
    __shared__ uint32_t tmem_base_sh;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int per_qt = a.Hq * a.B;
    const int qt = a.nt - 1 - static_cast<int>(blockIdx.x) / per_qt;  // longest rows first
    const int rem = static_cast<int>(blockIdx.x) % per_qt;
    const int h = rem % a.Hq, b = rem / a.Hq;
    const int g = h / a.G;
    const int q0 = qt * kTl;
    const int jt0 = a.window > 0 ? max(0, q0 - a.window + 1) / kTl : 0;
    const int nk = qt - jt0 + 1;

    if (warp == 0 && lane == 0) {
        mbar_init(&q_full, 1);
        mbar_init(&st_full, 1);
        mbar_init(&st_free, 8);   // one arrival per coefficient warp
        mbar_init(&ds_full, 8);
        mbar_init(&ds_free[0], 1);
        mbar_init(&ds_free[1], 1);
        mbar_init(&acc_done, 1);
        mbar_init(&mma_idle, 1);
        for (int s = 0; s < kDqStages; ++s) {
            mbar_init(&kv_full[s], 1);
            mbar_init(&kv_empty[s], 1);
        }
        fence_barrier_init();
    }
    if (warp == 1) tmem_alloc_512(&tmem_base_sh);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_sh;

    if (warp < 4) {
        reg_dealloc<64>();
        if (warp == 0 && lane == 0) {
            // --------------------------------------------------- TMA producer
            tma_prefetch_desc(&tq);
            tma_prefetch_desc(&tk);
            tma_prefetch_desc(&tv);
            tma_prefetch_desc(&tda);
            mbar_arrive_expect_tx(&q_full, 2 * kTileB);
            tma_load_4d(sQ, &tq, 0, h, q0, b, &q_full);
            tma_load_3d(sDA, &tda, 0, q0, b * a.Hq + h, &q_full);
            int issued = 0;
            bool ok = true;
            for (int n = 0; n < nk && ok; ++n) {
                const int s = n % kDqStages;
                if (n >= kDqStages &&
                    !(ok = mbar_wait(&kv_empty[s], ((n / kDqStages) - 1) & 1, a.status)))
                    break;
                uint8_t *st = sKV + s * 2 * kTileB;
                mbar_arrive_expect_tx(&kv_full[s], 2 * kTileB);
                tma_load_4d(st, &tk, 0, g, (jt0 + n) * kTl, b, &kv_full[s]);
                tma_load_4d(st + kTileB, &tv, 0, g, (jt0 + n) * kTl, b, &kv_full[s]);
                ++issued;
            }
            mbar_wait(&q_full, 0, a.status);
            for (int n = (issued > kDqStages ? issued - kDqStages : 0); n < issued; ++n)
                mbar_wait(&kv_full[n % kDqStages], (n / kDqStages) & 1, a.status);
        } else if (warp == 1 && lane == 0) {
            // ---------------------------------------------------- MMA issuer
            constexpr uint32_t idesc_s = idesc_bf16(kTl, kTl, false);     // Q K^T, dA V^T
            constexpr uint32_t idesc_dq = idesc_bf16(kTl, 64, true);      // dS K (K as MN-major B)
            const uint32_t hi = kSdescHi128B;
            const uint32_t q_lo = sdesc_lo(smem_u32(sQ), 16), da_lo = sdesc_lo(smem_u32(sDA), 16);
            bool ok = mbar_wait(&q_full, 0, a.status);
            auto kv_lo = [&](int s, int which, uint32_t lbo) {
                return sdesc_lo(smem_u32(sKV + s * 2 * kTileB + which * kTileB), lbo);
            };
            auto issue_dq = [&](int m) {
                if (!(ok = ok && mbar_wait(&ds_full, m & 1, a.status))) return;
                tc_fence_after();
                const int s = m % kDqStages;
                const uint32_t k_mn = kv_lo(s, 0, 8192);
#pragma unroll
                for (int kk = 0; kk < kTl / 16; ++kk)
                    mma_ts2(tmem + kColDQ, tmem + kColDS + 64 * (m & 1) + 8 * kk, k_mn + 128 * kk, hi,
                            idesc_dq, (m > 0 || kk > 0) ? 1u : 0u);
                tc_commit(&ds_free[m & 1]);
                tc_commit(&kv_empty[s]);
            };
            for (int n = 0; n < nk && ok; ++n) {
                const int s = n % kDqStages;
                if (!(ok = mbar_wait(&kv_full[s], (n / kDqStages) & 1, a.status))) break;
                if (n > 0 && !(ok = mbar_wait(&st_free, (n - 1) & 1, a.status))) break;
                tc_fence_after();
                const uint32_t k_k = kv_lo(s, 0, 16), v_k = kv_lo(s, 1, 16);
                mma_ss2<0>(tmem + kColS, q_lo, hi, k_k, hi, idesc_s);
#pragma unroll
                for (int kk = 1; kk < 4; ++kk)
                    mma_ss2<1>(tmem + kColS, q_lo + 2 * kk, hi, k_k + 2 * kk, hi, idesc_s);
                mma_ss2<0>(tmem + kColAV, da_lo, hi, v_k, hi, idesc_s);
#pragma unroll
                for (int kk = 1; kk < 4; ++kk)
                    mma_ss2<1>(tmem + kColAV, da_lo + 2 * kk, hi, v_k + 2 * kk, hi, idesc_s);
                tc_commit(&st_full);
                if (n > 0) issue_dq(n - 1);
            }
            if (ok && nk > 0) issue_dq(nk - 1);
            tc_commit(&acc_done);
            tc_commit(&mma_idle);
            mbar_wait(&mma_idle, 0, a.status);
        }
    } else {
        reg_alloc<208>();
        // ------------------------------------------------- coefficient threads
        const int wg = (warp - 4) >> 2;   // key half
        const int wq = warp & 3;
        const int t = 32 * wq + lane;     // row within the tile = TMEM lane
        const int i = q0 + t;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(32 * wq) << 16);
        const float4 *cr = reinterpret_cast<const float4 *>(
            a.coef + ((static_cast<size_t>(b) * a.Hq + h) * a.Tpad + i) * kBwdCoefWords);
        const float4 c0 = __ldg(cr), c1 = __ldg(cr + 1), c2 = __ldg(cr + 2);
        bool ok = true;
        for (int n = 0; n < nk; ++n) {
            const int jt = jt0 + n;
            ok = mbar_wait(&st_full, n & 1, a.status);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            tc_fence_after();
            uint32_t sr[2][32], ar[2][32];
            tmem_ld32(lane_base + kColS + 64 * wg, sr[0]);
            tmem_ld32(lane_base + kColS + 64 * wg + 32, sr[1]);
            tmem_ld32(lane_base + kColAV + 64 * wg, ar[0]);
            tmem_ld32(lane_base + kColAV + 64 * wg + 32, ar[1]);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&st_free);
            const bool masked = jt == qt || (a.window > 0 && jt * kTl < min(q0 + kTl, a.T) - a.window);
            const int kbase = jt * kTl + 64 * wg;
            uint32_t dp[32], unused[32];
            if (masked)
                pair_grads<true, false>(sr, ar, c0, c1, __float_as_int(c2.y) - kbase, i - kbase,
                                        unused, dp);
            else
                pair_grads<false, false>(sr, ar, c0, c1, 0, 0, unused, dp);
            // dS(n) goes to buffer n % 2: free once dQ(n-2) has read it.
            if (n > 1) {
                ok = mbar_wait(&ds_free[n & 1], ((n - 2) >> 1) & 1, a.status);
                if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                tc_fence_after();
            }
            uint32_t d0[16], d1[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                d0[e] = dp[e];
                d1[e] = dp[16 + e];
            }
            const uint32_t tds = lane_base + kColDS + 64 * (n & 1) + 32 * wg;
            tmem_st16(tds, d0);
            tmem_st16(tds + 16, d1);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&ds_full);
        }
        // Epilogue: 32 of the 64 dims of dQ per warpgroup, plus the argmax term
        // c dm k_{jmax} in fp32.
        if (ok) ok = mbar_wait(&acc_done, 0, a.status);
        if (__all_sync(0xffffffffu, ok) && nk > 0) {
            tc_fence_after();
            uint32_t o[32];
            tmem_ld32(lane_base + kColDQ + 32 * wg, o);
            tmem_wait_ld();
            const int jm = __float_as_int(c2.x);
            if (i < a.T) {
                float v[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) v[e] = __uint_as_float(o[e]);
                if (jm >= 0 && jm < a.T) {
                    const uint4 *kr = reinterpret_cast<const uint4 *>(
                        a.k + ((static_cast<size_t>(b) * a.T + jm) * a.Hkv + g) * kHeadDim + 32 * wg);
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const uint4 kk = __ldg(kr + c);
                        const uint32_t kw[4] = {kk.x, kk.y, kk.z, kk.w};
#pragma unroll
                        for (int x = 0; x < 4; ++x) {
                            v[8 * c + 2 * x] = fmaf(c1.w, __uint_as_float(kw[x] << 16), v[8 * c + 2 * x]);
                            v[8 * c + 2 * x + 1] =
                                fmaf(c1.w, __uint_as_float(kw[x] & 0xFFFF0000u), v[8 * c + 2 * x + 1]);
                        }
                    }
                }
                float4 *dst = reinterpret_cast<float4 *>(
                    a.dq + ((static_cast<size_t>(b) * a.T + i) * a.Hq + h) * kHeadDim + 32 * wg);
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    dst[c] = make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
            }
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


// -------------------------------------------------------- dQ pass, head pair ---
// The dQ pass for an even group size, in the forward's layout: one CTA per
// (128-row query tile, pair of query heads of one kv group, batch), both heads
// sharing every K/V tile.  Each key tile is taken in two 64-key halves: for
// each head, S and <dA, v> of one half at a time (N = 64) sit in tensor memory
// next to the head's dS (the whole tile, bf16) and its dQ accumulator, 256
// columns per head.  Each head has its own coefficient warpgroup, so one
// head's arithmetic overlaps the other head's products; one thread issues the
// score products (both heads, both halves) and another the dQ products.
constexpr int kDq2Stages = 4;
constexpr int kDq2Smem = 4 * kTileB + kDq2Stages * 2 * kTileB + 1024;  // 193 KB
constexpr uint32_t kC2S = 0, kC2AV = 64, kC2DS = 128, kC2DQ = 192;  // per head: + 256 * slot

__global__ void __launch_bounds__(384, 1)
bwd_dq2_tc_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                  const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tda,
                  const BwdTcArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024(smem_raw);
    uint8_t *sQ = smem;                    // Q of head slot 0, then slot 1
    uint8_t *sDA = smem + 2 * kTileB;      // dA of slot 0, then slot 1
    uint8_t *sKV = smem + 4 * kTileB;      // stage s: K at s * 2 tiles, V after it

    __shared__ __align__(8) uint64_t q_full, acc_done, mma_idle[2];
    __shared__ __align__(8) uint64_t st_full[2], st_free[2], ds_full[2], ds_free[2];
    __shared__ __align__(8) uint64_t kv_full[kDq2Stages], kv_empty[kDq2Stages];
    __shared__ uint32_t tmem_base_sh;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int npairs = a.Hq / 2;
    const int per_qt = npairs * a.B;
    const int qt = a.nt - 1 - static_cast<int>(blockIdx.x) / per_qt;  // longest rows first
    const int rem = static_cast<int>(blockIdx.x) % per_qt;
    const int h0 = 2 * (rem % npairs), b = rem / npairs;
    const int g = h0 / a.G;
    const int q0 = qt * kTl;
    const int jt0 = a.window > 0 ? max(0, q0 - a.window + 1) / kTl : 0;
    const int nk = qt - jt0 + 1;

    if (warp == 0 && lane == 0) {
        mbar_init(&q_full, 1);
        mbar_init(&acc_done, 1);
        mbar_init(&mma_idle[0], 1);
        mbar_init(&mma_idle[1], 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&st_full[i], 1);
            mbar_init(&st_free[i], 4);  // one arrival per warp of the head's warpgroup
            mbar_init(&ds_full[i], 4);
            mbar_init(&ds_free[i], 1);
        }
        for (int s = 0; s < kDq2Stages; ++s) {
            mbar_init(&kv_full[s], 1);
            mbar_init(&kv_empty[s], 2);  // one commit from each issuer
        }
        fence_barrier_init();
    }
    if (warp == 1) tmem_alloc_512(&tmem_base_sh);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_sh;

    if (warp < 4) {
        reg_dealloc<64>();
        if (warp == 0 && lane == 0) {
            // --------------------------------------------------- TMA producer
            tma_prefetch_desc(&tq);
            tma_prefetch_desc(&tk);
            tma_prefetch_desc(&tv);
            tma_prefetch_desc(&tda);
            mbar_arrive_expect_tx(&q_full, 4 * kTileB);
            for (int i = 0; i < 2; ++i) {
                tma_load_4d(sQ + i * kTileB, &tq, 0, h0 + i, q0, b, &q_full);
                tma_load_3d(sDA + i * kTileB, &tda, 0, q0, b * a.Hq + h0 + i, &q_full);
            }
            int issued = 0;
            bool ok = true;
            for (int n = 0; n < nk && ok; ++n) {
                const int s = n % kDq2Stages;
                if (n >= kDq2Stages &&
                    !(ok = mbar_wait(&kv_empty[s], ((n / kDq2Stages) - 1) & 1, a.status)))
                    break;
                uint8_t *st = sKV + s * 2 * kTileB;
                mbar_arrive_expect_tx(&kv_full[s], 2 * kTileB);
                tma_load_4d(st, &tk, 0, g, (jt0 + n) * kTl, b, &kv_full[s]);
                tma_load_4d(st + kTileB, &tv, 0, g, (jt0 + n) * kTl, b, &kv_full[s]);
                ++issued;
            }
            mbar_wait(&q_full, 0, a.status);
            for (int n = (issued > kDq2Stages ? issued - kDq2Stages : 0); n < issued; ++n)
                mbar_wait(&kv_full[n % kDq2Stages], (n / kDq2Stages) & 1, a.status);
        } else if ((warp == 1 || warp == 2) && lane == 0) {
            const uint32_t hi = kSdescHi128B;
            auto kv_lo = [&](int s, int which, uint32_t lbo) {
                return sdesc_lo(smem_u32(sKV + s * 2 * kTileB + which * kTileB), lbo);
            };
            bool ok = true;
            if (warp == 1) {
                // ------------------- score issuer: S and <dA, v> per head and half
                constexpr uint32_t idesc_h = idesc_bf16(kTl, 64, false);  // N = 64 keys
                ok = mbar_wait(&q_full, 0, a.status);
                for (int n = 0; n < nk && ok; ++n) {
                    const int s = n % kDq2Stages;
                    if (!(ok = mbar_wait(&kv_full[s], (n / kDq2Stages) & 1, a.status))) break;
                    for (int half = 0; half < 2 && ok; ++half) {
                        for (int i = 0; i < 2 && ok; ++i) {
                            const int step = 2 * n + half;
                            if (step > 0 && !(ok = mbar_wait(&st_free[i], (step - 1) & 1, a.status)))
                                break;
                            tc_fence_after();
                            // keys 64 half .. + 63: 64 rows of 128 B further into the tile
                            const uint32_t k_k = kv_lo(s, 0, 16) + 512 * half;
                            const uint32_t v_k = kv_lo(s, 1, 16) + 512 * half;
                            const uint32_t q_k = sdesc_lo(smem_u32(sQ + i * kTileB), 16);
                            const uint32_t a_k = sdesc_lo(smem_u32(sDA + i * kTileB), 16);
                            const uint32_t col = tmem + 256 * i;
                            mma_ss2<0>(col + kC2S, q_k, hi, k_k, hi, idesc_h);
#pragma unroll
                            for (int kk = 1; kk < 4; ++kk)
                                mma_ss2<1>(col + kC2S, q_k + 2 * kk, hi, k_k + 2 * kk, hi, idesc_h);
                            mma_ss2<0>(col + kC2AV, a_k, hi, v_k, hi, idesc_h);
#pragma unroll
                            for (int kk = 1; kk < 4; ++kk)
                                mma_ss2<1>(col + kC2AV, a_k + 2 * kk, hi, v_k + 2 * kk, hi, idesc_h);
                            tc_commit(&st_full[i]);
                        }
                    }
                    if (ok) tc_commit(&kv_empty[s]);
                }
            } else {
                // ------------------------------------ dQ issuer: dQ += dS K per head
                constexpr uint32_t idesc_dq = idesc_bf16(kTl, 64, true);  // K as MN-major B
                for (int n = 0; n < nk && ok; ++n) {
                    const int s = n % kDq2Stages;
                    if (!(ok = mbar_wait(&kv_full[s], (n / kDq2Stages) & 1, a.status))) break;
                    const uint32_t k_mn = kv_lo(s, 0, 8192);
                    for (int i = 0; i < 2 && ok; ++i) {
                        if (!(ok = mbar_wait(&ds_full[i], n & 1, a.status))) break;
                        tc_fence_after();
                        const uint32_t col = tmem + 256 * i;
#pragma unroll
                        for (int kk = 0; kk < kTl / 16; ++kk)
                            mma_ts2(col + kC2DQ, col + kC2DS + 8 * kk, k_mn + 128 * kk, hi, idesc_dq,
                                    (n > 0 || kk > 0) ? 1u : 0u);
                        tc_commit(&ds_free[i]);
                    }
                    if (ok) tc_commit(&kv_empty[s]);
                }
                tc_commit(&acc_done);
            }
            // Every MMA this thread issued completes before tensor memory is freed.
            tc_commit(&mma_idle[warp - 1]);
            mbar_wait(&mma_idle[warp - 1], 0, a.status);
        }
    } else {
        reg_alloc<208>();
        // ------------------------------- coefficient warpgroups, one per head
        const int slot = (warp - 4) >> 2;
        const int wq = warp & 3;
        const int t = 32 * wq + lane;     // row within the tile = TMEM lane
        const int h = h0 + slot, i = q0 + t;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(32 * wq) << 16) + 256 * slot;
        const float4 *cr = reinterpret_cast<const float4 *>(
            a.coef + ((static_cast<size_t>(b) * a.Hq + h) * a.Tpad + i) * kBwdCoefWords);
        const float4 c0 = __ldg(cr), c1 = __ldg(cr + 1), c2 = __ldg(cr + 2);
        bool ok = true;
        for (int n = 0; n < nk && ok; ++n) {
            const int jt = jt0 + n;
            const bool masked = jt == qt || (a.window > 0 && jt * kTl < min(q0 + kTl, a.T) - a.window);
            for (int half = 0; half < 2; ++half) {
                const int step = 2 * n + half;
                ok = mbar_wait(&st_full[slot], step & 1, a.status);
                if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                tc_fence_after();
                uint32_t sr[2][32], ar[2][32];
                tmem_ld32(lane_base + kC2S, sr[0]);
                tmem_ld32(lane_base + kC2S + 32, sr[1]);
                tmem_ld32(lane_base + kC2AV, ar[0]);
                tmem_ld32(lane_base + kC2AV + 32, ar[1]);
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&st_free[slot]);
                const int kbase = jt * kTl + 64 * half;
                uint32_t dp[32], unused[32];
                if (masked)
                    pair_grads<true, false>(sr, ar, c0, c1, __float_as_int(c2.y) - kbase, i - kbase,
                                            unused, dp);
                else
                    pair_grads<false, false>(sr, ar, c0, c1, 0, 0, unused, dp);
                // dS of the previous tile consumed by its dQ product before the first half.
                if (half == 0 && n > 0) {
                    ok = mbar_wait(&ds_free[slot], (n - 1) & 1, a.status);
                    if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                    tc_fence_after();
                }
                uint32_t d0[16], d1[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    d0[e] = dp[e];
                    d1[e] = dp[16 + e];
                }
                tmem_st16(lane_base + kC2DS + 32 * half, d0);
                tmem_st16(lane_base + kC2DS + 32 * half + 16, d1);
                tmem_wait_st();
                tc_fence_before();
                if (half == 1) {
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&ds_full[slot]);
                }
            }
        }
        // Epilogue: dQ of row i and head h, plus the argmax term c dm k_{jmax} in fp32.
        if (ok) ok = mbar_wait(&acc_done, 0, a.status);
        if (__all_sync(0xffffffffu, ok) && nk > 0) {
            tc_fence_after();
            uint32_t o[2][32];
            tmem_ld32(lane_base + kC2DQ, o[0]);
            tmem_ld32(lane_base + kC2DQ + 32, o[1]);
            tmem_wait_ld();
            const int jm = __float_as_int(c2.x);
            if (i < a.T) {
                float v[64];
#pragma unroll
                for (int e = 0; e < 64; ++e) v[e] = __uint_as_float(o[e >> 5][e & 31]);
                if (jm >= 0 && jm < a.T) {
                    const uint4 *kr = reinterpret_cast<const uint4 *>(
                        a.k + ((static_cast<size_t>(b) * a.T + jm) * a.Hkv + g) * kHeadDim);
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const uint4 kk = __ldg(kr + c);
                        const uint32_t kw[4] = {kk.x, kk.y, kk.z, kk.w};
#pragma unroll
                        for (int x = 0; x < 4; ++x) {
                            v[8 * c + 2 * x] = fmaf(c1.w, __uint_as_float(kw[x] << 16), v[8 * c + 2 * x]);
                            v[8 * c + 2 * x + 1] =
                                fmaf(c1.w, __uint_as_float(kw[x] & 0xFFFF0000u), v[8 * c + 2 * x + 1]);
                        }
                    }
                }
                float4 *dst = reinterpret_cast<float4 *>(
                    a.dq + ((static_cast<size_t>(b) * a.T + i) * a.Hq + h) * kHeadDim);
#pragma unroll
                for (int c = 0; c < 16; ++c)
                    dst[c] = make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
            }
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

// A second stream per device for the dQ pass, which depends on the dK/dV
// pass for nothing: the two run side by side, so the dQ CTAs fill the SMs
// that the dK/dV pass's last wave leaves idle.  The mutex keeps one caller's
// fork (record, wait) and join from interleaving with another's.
struct SideStream {
    cudaStream_t s = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
    std::mutex mu;
    bool ready = false;
};

SideStream *side_stream(int dev) {
    static SideStream ss[64];
    static std::mutex init_mu;
    if (dev < 0 || dev >= 64) return nullptr;
    SideStream &x = ss[dev];
    std::lock_guard<std::mutex> lk(init_mu);
    if (!x.ready) {
        if (cudaStreamCreateWithFlags(&x.s, cudaStreamNonBlocking) != cudaSuccess ||
            cudaEventCreateWithFlags(&x.fork, cudaEventDisableTiming) != cudaSuccess ||
            cudaEventCreateWithFlags(&x.join, cudaEventDisableTiming) != cudaSuccess)
            return nullptr;
        x.ready = true;
    }
    return &x;
}

}  // namespace

cudaError_t launch_bwd_tc(const BwdLaunch &l, const float *coef, const void *dab) {
    static std::atomic<uint64_t> configured{0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = 1ull << (dev & 63);
    if (!(configured.load() & bit)) {
        e = cudaFuncSetAttribute(bwd_dkdv_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kDkdvSmem);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(bwd_dq_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kDqSmem);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(bwd_dq2_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kDq2Smem);
        if (e != cudaSuccess) return e;
        // setmaxnreg hands out only the registers the block was launched with:
        // 64 x 128 (producer, issuer) + 208 x 256 (coefficient threads) must fit.
        const void *fns[] = {reinterpret_cast<const void *>(bwd_dkdv_tc_kernel),
                             reinterpret_cast<const void *>(bwd_dq_tc_kernel),
                             reinterpret_cast<const void *>(bwd_dq2_tc_kernel)};
        for (const void *f : fns) {
            cudaFuncAttributes fa;
            e = cudaFuncGetAttributes(&fa, f);
            if (e != cudaSuccess) return e;
            if (static_cast<long long>(fa.numRegs) * 384 < 64ll * 128 + 208ll * 256)
                return cudaErrorInvalidConfiguration;
        }
        configured.fetch_or(bit);
    }
    const int Tpad = (l.T + kTl - 1) / kTl * kTl;
    CUtensorMap tq, tk, tv, tda;
    const uint32_t box4[4] = {kHeadDim, 1, kTl, 1};
    {
        const uint64_t dims[4] = {kHeadDim, (uint64_t)l.Hq, (uint64_t)l.T, (uint64_t)l.B};
        const uint64_t str[3] = {kHeadDim * 2ull, (uint64_t)l.Hq * kHeadDim * 2,
                                 (uint64_t)l.T * l.Hq * kHeadDim * 2};
        if (encode_tiled(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(l.q), dims,
                         str, box4, CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    {
        const uint64_t dims[4] = {kHeadDim, (uint64_t)l.Hkv, (uint64_t)l.T, (uint64_t)l.B};
        const uint64_t str[3] = {kHeadDim * 2ull, (uint64_t)l.Hkv * kHeadDim * 2,
                                 (uint64_t)l.T * l.Hkv * kHeadDim * 2};
        if (encode_tiled(&tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(l.k), dims,
                         str, box4, CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS ||
            encode_tiled(&tv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(l.v), dims,
                         str, box4, CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    {
        // dA as bf16 [B*Hq][Tpad][64]: tiles of 128 rows of one (batch, head).
        const uint64_t dims[3] = {kHeadDim, (uint64_t)Tpad, (uint64_t)l.B * l.Hq};
        const uint64_t str[2] = {kHeadDim * 2ull, (uint64_t)Tpad * kHeadDim * 2};
        const uint32_t box3[3] = {kHeadDim, kTl, 1};
        if (encode_tiled(&tda, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(dab), dims,
                         str, box3, CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    BwdTcArgs a;
    a.coef = coef;
    a.k = static_cast<const __nv_bfloat16 *>(l.k);
    a.dq = l.dq; a.dk = l.dk; a.dv = l.dv;
    a.status = l.status;
    a.B = l.B; a.T = l.T; a.Tpad = Tpad; a.Hq = l.Hq; a.Hkv = l.Hkv; a.G = l.Hq / l.Hkv;
    a.nt = Tpad / kTl;
    a.window = l.window > 0 && l.window < l.T ? l.window : 0;
    const long long kv_ctas = static_cast<long long>(a.nt) * l.Hkv * l.B;
    const long long q_ctas = static_cast<long long>(a.nt) * l.Hq * l.B;
    if (kv_ctas > 0x7fffffffll || q_ctas > 0x7fffffffll) return cudaErrorInvalidValue;
    SideStream *ss = side_stream(dev);
    if (!ss) return cudaErrorUnknown;
    std::lock_guard<std::mutex> lk(ss->mu);
    e = cudaEventRecord(ss->fork, l.stream);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(ss->s, ss->fork, 0);
    if (e != cudaSuccess) return e;
    bwd_dkdv_tc_kernel<<<static_cast<unsigned>(kv_ctas), 384, kDkdvSmem, l.stream>>>(tq, tk, tv,
                                                                                     tda, a);
    if (a.G % 2 == 0)  // head pairs share each K/V tile
        bwd_dq2_tc_kernel<<<static_cast<unsigned>(q_ctas / 2), 384, kDq2Smem, ss->s>>>(tq, tk, tv,
                                                                                        tda, a);
    else
        bwd_dq_tc_kernel<<<static_cast<unsigned>(q_ctas), 384, kDqSmem, ss->s>>>(tq, tk, tv, tda, a);
    e = cudaGetLastError();
    // Join even after a failed launch, so that the caller's stream never runs
    // ahead of work already queued on the side stream.
    const cudaError_t ej = cudaEventRecord(ss->join, ss->s);
    const cudaError_t ew = ej == cudaSuccess ? cudaStreamWaitEvent(l.stream, ss->join, 0) : ej;
    count_launches(2);
    return e != cudaSuccess ? e : ew;
}

}  // namespace polar
