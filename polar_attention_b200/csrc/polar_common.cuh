// polar_common.cuh -- device helpers shared by the library's kernels:
// bounded mbarrier waits, TMA / bulk-copy and tcgen05 PTX wrappers, and the
// Polar Attention epilogue (participation ratio, null floor, gate, count).
//
// Method: "ATMA: Length-Invariant Language Modeling via Polar Attention and
// Gated-Delta Compression Memory", gist.science technical summary, section 2.1
// (direction channel, magnitude channel) and section 2.2 (fused kernel with
// streaming accumulators and squared correction factors; GQA paged decode).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "polar_attn.h"

namespace polar {

constexpr int kHeadDim = 64;
constexpr int kPage = 64;               // tokens per KV page
constexpr float kLog2e = 1.4426950408889634f;
// Lazy rescale threshold, log2 units: the reference max of the streaming
// softmax only moves when a new logit exceeds it by more than 2^8, so every
// weight stays <= 256 and its square <= 65536 (safe in fp32).  Exact: n_eff and
// the direction are invariant to the common scale of l, l2 and acc.
constexpr float kRescaleThreshold = 8.0f;
// Budget of a bounded wait, in SM clock cycles (about one second at 2 GHz).
constexpr long long kWaitBudget = 1ll << 31;

// ---------------------------------------------------------------- status ---

__device__ __forceinline__ void record_error(int *status, int code) {
    if (status) atomicCAS(status, 0, code);
}

// ------------------------------------------------------------- mbarrier ---

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Waits for the phase with the given parity to complete, for at most
// kWaitBudget cycles.  Returns false (and records POLAR_ERR_TIMEOUT) on
// timeout; never traps.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, int *status) {
    const uint32_t a = smem_u32(bar);
    if (mbar_try_wait(a, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try_wait(a, parity)) {
        if (clock64() - t0 > kWaitBudget) {
            record_error(status, POLAR_ERR_TIMEOUT);
            return false;
        }
    }
    return true;
}

// ------------------------------------------------------------------- TMA ---

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 2D tiled TMA load (no multicast) into this CTA's shared memory.
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y,
                                            uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

// 4D tiled TMA load (no multicast).
__device__ __forceinline__ void tma_load_4d(void *dst, const CUtensorMap *map, int x, int y,
                                            int z, int w, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(w),
        "r"(smem_u32(bar))
        : "memory");
}

// ------------------------------------------------------------- math ------

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// Length temperature tau(n) = 1 + alpha*ln(n/L) for n > L, else 1
// ("Length Temperature ... to sharpen distributions as context grows").
__device__ __forceinline__ float length_temperature(float n, float alpha, float L) {
    return n > L ? 1.0f + alpha * logf(n / L) : 1.0f;
}

// The magnitude channel's scalar for one row, from its streaming state.
//   l, l2  : sum_j w_j and sum_j w_j^2 with w_j = exp(z_j - m) for any common m
//   m_raw  : max_j <q, k_j>;  s1, s2: sum_j <q,k_j> and sum_j <q,k_j>^2
//   c      : logit scale times length temperature (z = c*<q,k>), n: visible keys
// n_eff = l^2/l2 (inverse Simpson index, clamped to [1, n]); the null floor
// z0 = mu + sigma*sqrt(2 ln n) uses the population mean/std of the logits;
// gate = sigmoid(beta*(max z - z0)); returns gate*tanh(ln n_eff / ln L).
__device__ __forceinline__ float polar_magnitude(float l, float l2, float m_raw, float s1,
                                                 float s2, float c, float n, float beta,
                                                 float inv_ln_L, float *neff_out) {
    float ne = (l * l) / l2;
    ne = fminf(fmaxf(ne, 1.0f), n);
    const float mean = s1 / n;
    const float var = fmaxf(s2 / n - mean * mean, 0.0f);
    const float z0 = c * (mean + sqrtf(var) * sqrtf(2.0f * logf(n)));
    const float gate = 1.0f / (1.0f + expf(-beta * (c * m_raw - z0)));
    *neff_out = ne;
    return gate * tanhf(logf(ne) * inv_ln_L);
}

template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
    return __bfloat162float(x);
}

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

}  // namespace polar
