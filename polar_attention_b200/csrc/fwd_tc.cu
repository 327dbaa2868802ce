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
// extent.  Warp roles (12 warps):
//   warp 0      TMA producer: Q tiles once, then K/V tiles into a 4-stage ring
//   warp 1      tensor-memory allocator and single-thread MMA issuer
//   warps 2-3   idle
//   warps 4-7   softmax warpgroup for head slot 0 (TMEM lanes 0-127)
//   warps 8-11  softmax warpgroup for head slot 1
// Tensor memory (512 columns): S0 S1 (128 fp32 columns each), P0 P1 (128 bf16
// packed in 64 columns each), O0 O1 (64 fp32 columns each).
// Issue order of the MMA thread, per key tile j:
//   PV0(j), S0(j+1), PV1(j), S1(j+1)
// so the tensor core computes one head's next scores while the other head's
// softmax runs.  A tcgen05.commit after S_i(j+1) also covers PV_i(j), which
// lets softmax i rescale O_i in place before it releases P_i(j+1).
#include <atomic>

#include "polar_attn_selftest.h"
#include "polar_common.cuh"
#include "polar_internal.h"

namespace polar {
namespace {

constexpr int kBM = 128;               // query rows per head slot
constexpr int kBN = 128;               // keys per tile
constexpr int kStagesKV = 4;           // K/V ring depth
constexpr int kTileBytes = 128 * 128;  // 128 rows x 64 bf16
constexpr int kThreads = 384;
constexpr int kSmemBytes = (2 + 2 * kStagesKV) * kTileBytes + 1024;

// Tensor-memory column map.
constexpr uint32_t kColS0 = 0, kColS1 = 128, kColP0 = 256, kColP1 = 320, kColO0 = 384,
                   kColO1 = 448;

// ---------------------------------------------------------------- tcgen05 --

__device__ __forceinline__ void tmem_alloc_512(uint32_t *dst_smem) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(
                     smem_u32(dst_smem))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_512(uint32_t taddr) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(taddr) : "memory");
}

// Register rebalancing between warpgroups (must be executed by all four warps
// of a warpgroup).  Budget: launched at 168 per thread x 384 threads = 64512;
// the producer/MMA warpgroup drops to 64 and the two softmax warpgroups rise to
// 216: 64*128 + 216*256 = 63488, within the launch total.
template <int N>
__device__ __forceinline__ void reg_dealloc() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void reg_alloc() {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, kind::f16 (bf16 in, fp32 accumulate).
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem].
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

#define POLAR_R32(r)                                                                      \
    "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),   \
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),        \
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),     \
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),     \
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),     \
        "=r"(r[31])

// 32 lanes x 32 consecutive 32-bit columns: thread t of the warp gets lane
// (warp's quarter base + t), columns taddr .. taddr + 31.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
        "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : POLAR_R32(r)
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
        "%13,%14,%15,%16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15])
        : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
        "%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(
            taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
        "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
        "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

// Shared-memory matrix descriptor for a 128B-swizzled tile (rows of 128
// bytes, 8-row groups 1024 bytes apart): start address, leading and stride
// byte offsets, descriptor version 1, layout SWIZZLE_128B.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4) |
           (static_cast<uint64_t>(lbo >> 4) << 16) | (static_cast<uint64_t>(sbo >> 4) << 32) |
           (1ull << 46) | (2ull << 61);
}

// Instruction descriptor, kind::f16: bf16 A and B, fp32 D, dense.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool b_mn_major) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(b_mn_major) << 16) |
           (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// ----------------------------------------------- packed fp32 (f32x2) math --

__device__ __forceinline__ float2 f2_add(float2 a, float2 b) {
    float2 d;
    asm("add.rn.f32x2 %0, %1, %2;"
        : "=l"(reinterpret_cast<uint64_t &>(d))
        : "l"(reinterpret_cast<const uint64_t &>(a)), "l"(reinterpret_cast<const uint64_t &>(b)));
    return d;
}

__device__ __forceinline__ float2 f2_fma(float2 a, float2 b, float2 c) {
    float2 d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;"
        : "=l"(reinterpret_cast<uint64_t &>(d))
        : "l"(reinterpret_cast<const uint64_t &>(a)), "l"(reinterpret_cast<const uint64_t &>(b)),
          "l"(reinterpret_cast<const uint64_t &>(c)));
    return d;
}

__device__ __forceinline__ float max3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

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

#ifndef POLAR_TC_POLY_MASK
// Which of every 16 exponential pairs of a full tile go to the polynomial
// (bit e set: pair e); the rest use MUFU ex2.  0x2222 = 4 of 16 (one quarter).
#define POLAR_TC_POLY_MASK 0x2222
#endif

// Row statistics of one 128-key tile of S (raw dots, one row per thread):
// max, sum and sum of squares over the visible keys.  Independent partial
// accumulators keep the dependency chains short.  kDiag: the tile holds the
// row's own position t; keys after it are invisible and are set to -inf in sr.
template <bool kDiag>
__device__ __forceinline__ void row_stats(uint32_t (&sr)[4][32], int t, float &tmax, float &ts1,
                                          float &ts2) {
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
            const bool vis = e <= t;
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
// (for l and l2), and the bf16 P tile written to tensor memory for the PV MMA.
// kPoly: the pairs selected by POLAR_TC_POLY_MASK use the FMA-pipe polynomial
// (full tiles only; the diagonal tile's -inf entries use ex2, which gives 0).
template <bool kPoly>
__device__ __forceinline__ void row_weights(const uint32_t (&sr)[4][32], float2 sc2, float neg_m,
                                            uint32_t tP, float &tl, float &tl2) {
    const float2 nm = make_float2(neg_m, neg_m);
    float2 la[2], l2a[2];
    la[0] = la[1] = l2a[0] = l2a[1] = make_float2(0.f, 0.f);
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
        uint32_t pk[16];
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
            pk[e] = pack_bf16(p.x, p.y);
        }
        tmem_st16(tP + 16 * cc, pk);
    }
    const float2 sl = f2_add(la[0], la[1]), sl2 = f2_add(l2a[0], l2a[1]);
    tl = sl.x + sl.y;
    tl2 = sl2.x + sl2.y;
}

struct TcArgs {
    const float *u;
    __nv_bfloat16 *out;
    float *neff;
    int *status;
    int B, T, Hq, Hkv, nqt, npairs;
    float s, alpha, L, beta, inv_ln_L;
};

__global__ void __launch_bounds__(kThreads, 1)
fwd_tc_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
              const __grid_constant__ CUtensorMap tv, const TcArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = smem;                           // 2 tiles
    uint8_t *sK = smem + 2 * kTileBytes;          // kStagesKV tiles
    uint8_t *sV = sK + kStagesKV * kTileBytes;    // kStagesKV tiles

    __shared__ __align__(8) uint64_t q_full, kv_full[kStagesKV], kv_empty[kStagesKV];
    __shared__ __align__(8) uint64_t s_full[2], p_full[2], o_done[2], mma_done;
    __shared__ uint32_t tmem_base_sh;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // Work tile: heaviest query tiles first (longest causal rows).
    const int per_qt = a.npairs * a.B;
    const int qt = a.nqt - 1 - static_cast<int>(blockIdx.x) / per_qt;
    const int rem = static_cast<int>(blockIdx.x) % per_qt;
    const int pair = rem % a.npairs, b = rem / a.npairs;
    const int h0 = 2 * pair;
    const int g = h0 / (a.Hq / a.Hkv);
    const int q0 = qt * kBM;
    const int nkv = qt + 1;  // key tiles 0..qt are (partly) visible

    if (warp == 0 && lane == 0) {
        mbar_init(&q_full, 1);
        for (int st = 0; st < kStagesKV; ++st) {
            mbar_init(&kv_full[st], 1);
            mbar_init(&kv_empty[st], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s_full[i], 1);
            mbar_init(&p_full[i], kBM);
            mbar_init(&o_done[i], 1);
        }
        mbar_init(&mma_done, 1);
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
                tma_load_4d(sK + st * kTileBytes, &tk, 0, g, j * kBN, b, &kv_full[st]);
                tma_load_4d(sV + st * kTileBytes, &tv, 0, g, j * kBN, b, &kv_full[st]);
                ++issued;
            }
            // Every copy this thread started lands before shared memory is released.
            mbar_wait(&q_full, 0, a.status);
            for (int j = (issued > kStagesKV ? issued - kStagesKV : 0); j < issued; ++j)
                mbar_wait(&kv_full[j % kStagesKV], (j / kStagesKV) & 1, a.status);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_qk = idesc_bf16(kBM, kBN, false);
            constexpr uint32_t idesc_pv = idesc_bf16(kBM, kHeadDim, true);
            const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK), sVa = smem_u32(sV);
            const uint32_t colS[2] = {kColS0, kColS1}, colP[2] = {kColP0, kColP1},
                           colO[2] = {kColO0, kColO1};
            auto issue_s = [&](int i, int j) {
                const uint32_t qa = sQa + i * kTileBytes, ka = sKa + (j % kStagesKV) * kTileBytes;
#pragma unroll
                for (int kk = 0; kk < kHeadDim / 16; ++kk)
                    mma_ss(tmem + colS[i], sw128_desc(qa + 32 * kk, 16, 1024),
                           sw128_desc(ka + 32 * kk, 16, 1024), idesc_qk, kk > 0);
                tc_commit(&s_full[i]);
            };
            auto issue_pv = [&](int i, int j) {
                const uint32_t va = sVa + (j % kStagesKV) * kTileBytes;
#pragma unroll
                for (int kk = 0; kk < kBN / 16; ++kk)
                    mma_ts(tmem + colO[i], tmem + colP[i] + 8 * kk,
                           sw128_desc(va + 2048 * kk, 8192, 1024), idesc_pv, (j > 0 || kk > 0));
            };
            bool ok = mbar_wait(&q_full, 0, a.status) && mbar_wait(&kv_full[0], 0, a.status);
            if (ok) {
                tc_fence_after();
                issue_s(0, 0);
                issue_s(1, 0);
            }
            for (int j = 0; j < nkv && ok; ++j) {
                ok = mbar_wait(&p_full[0], j & 1, a.status);
                if (!ok) break;
                tc_fence_after();
                issue_pv(0, j);
                if (j + 1 < nkv) {
                    ok = mbar_wait(&kv_full[(j + 1) % kStagesKV], ((j + 1) / kStagesKV) & 1, a.status);
                    if (!ok) break;
                    tc_fence_after();
                    issue_s(0, j + 1);
                } else {
                    tc_commit(&o_done[0]);
                }
                ok = mbar_wait(&p_full[1], j & 1, a.status);
                if (!ok) break;
                tc_fence_after();
                issue_pv(1, j);
                tc_commit(&kv_empty[j % kStagesKV]);
                if (j + 1 < nkv)
                    issue_s(1, j + 1);
                else
                    tc_commit(&o_done[1]);
            }
            // All MMAs this thread issued complete before tensor memory is freed.
            tc_commit(&mma_done);
            mbar_wait(&mma_done, 0, a.status);
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
        const float n = static_cast<float>(row + 1);
        const float c = a.s * length_temperature(n, a.alpha, a.L);
        const float cl2 = c * kLog2e;

        float m_ref = -INFINITY, m_raw = -INFINITY, l = 0.f, l2 = 0.f, s1 = 0.f, s2 = 0.f;
        const float2 sc2 = make_float2(cl2, cl2);
        bool ok = true;
        for (int j = 0; j < nkv; ++j) {
            ok = mbar_wait(&s_full[slot], j & 1, a.status);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            tc_fence_after();
            uint32_t sr[4][32];
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) tmem_ld32(tS + 32 * cc, sr[cc]);
            tmem_wait_ld();
            const bool diag = (j == nkv - 1);
            float tmax, ts1, ts2;
            if (diag)
                row_stats<true>(sr, t, tmax, ts1, ts2);
            else
                row_stats<false>(sr, t, tmax, ts1, ts2);
            s1 += ts1;
            s2 += ts2;
            m_raw = fmaxf(m_raw, tmax);
            const float zmax = tmax * cl2;
            const bool need = zmax > m_ref + kRescaleThreshold;
            float r = 1.f;
            if (need) {
                r = ex2(m_ref - zmax);  // 0 on the first tile
                l *= r;
                l2 *= r * r;
                m_ref = zmax;
            }
            float tl, tl2;
            if (diag)
                row_weights<false>(sr, sc2, -m_ref, tP, tl, tl2);
            else
                row_weights<true>(sr, sc2, -m_ref, tP, tl, tl2);
            l += tl;
            l2 += tl2;
            // Rescale the output accumulator when this row's reference max moved.
            // Safe: S(j) landing implies PV(j-1) has completed (one commit covers both).
            if (j > 0 && __any_sync(0xffffffffu, need)) {
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
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&p_full[slot]);
        }
        if (ok) ok = mbar_wait(&o_done[slot], 0, a.status);
        if (__all_sync(0xffffffffu, ok)) {
            tc_fence_after();
            uint32_t o[2][32];
            tmem_ld32(tO, o[0]);
            tmem_ld32(tO + 32, o[1]);
            tmem_wait_ld();
            if (row < a.T) {
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
                const float inv = 1.0f / fmaxf(sqrtf(nrm), 1e-30f);
                const float4 *u4 = reinterpret_cast<const float4 *>(a.u + static_cast<size_t>(h) * kHeadDim);
                uint4 *dst = reinterpret_cast<uint4 *>(
                    a.out + ((static_cast<size_t>(b) * a.T + row) * a.Hq + h) * kHeadDim);
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

__global__ void selftest_exp2_kernel(const float2 *x, float2 *poly, float2 *mufu, int npairs) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= npairs) return;
    const float2 v = x[i];
    poly[i] = exp2_poly2(v);
    mufu[i] = make_float2(ex2(v.x), ex2(v.y));
}

}  // namespace

cudaError_t launch_fwd_tc(const FwdLaunch &a) {
    const int G = a.Hq / a.Hkv;
    if (a.dtype != POLAR_BF16 || G % 2 != 0) return cudaErrorNotSupported;
    static std::atomic<uint64_t> configured{0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = 1ull << (dev & 63);
    if (!(configured.load() & bit)) {
        e = cudaFuncSetAttribute(fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kSmemBytes);
        if (e != cudaSuccess) return e;
        configured.fetch_or(bit);
    }
    // [B, T, H, 64] bf16 as a 4-D tensor (d, head, t, b); tiles of 128 rows x 64.
    CUtensorMap tq, tk, tv;
    const uint32_t box[4] = {kHeadDim, 1, 128, 1};
    {
        const uint64_t dims[4] = {kHeadDim, (uint64_t)a.Hq, (uint64_t)a.T, (uint64_t)a.B};
        const uint64_t str[3] = {kHeadDim * 2ull, (uint64_t)a.Hq * kHeadDim * 2,
                                 (uint64_t)a.T * a.Hq * kHeadDim * 2};
        if (encode_tiled(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(a.q), dims, str,
                         box, CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    {
        const uint64_t dims[4] = {kHeadDim, (uint64_t)a.Hkv, (uint64_t)a.T, (uint64_t)a.B};
        const uint64_t str[3] = {kHeadDim * 2ull, (uint64_t)a.Hkv * kHeadDim * 2,
                                 (uint64_t)a.T * a.Hkv * kHeadDim * 2};
        if (encode_tiled(&tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(a.k), dims, str,
                         box, CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS ||
            encode_tiled(&tv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(a.v), dims, str,
                         box, CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    TcArgs ta;
    ta.u = a.u;
    ta.out = static_cast<__nv_bfloat16 *>(a.out);
    ta.neff = a.neff;
    ta.status = a.status;
    ta.B = a.B; ta.T = a.T; ta.Hq = a.Hq; ta.Hkv = a.Hkv;
    ta.nqt = (a.T + kBM - 1) / kBM;
    ta.npairs = a.Hq / 2;
    ta.s = a.s; ta.alpha = a.alpha; ta.L = static_cast<float>(a.L); ta.beta = a.beta;
    ta.inv_ln_L = 1.0f / logf(static_cast<float>(a.L));
    const long long ctas = static_cast<long long>(ta.nqt) * ta.npairs * a.B;
    if (ctas <= 0) return cudaSuccess;
    if (ctas > 0x7fffffffll) return cudaErrorInvalidValue;
    fwd_tc_kernel<<<static_cast<unsigned>(ctas), kThreads, kSmemBytes, a.stream>>>(tq, tk, tv, ta);
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
