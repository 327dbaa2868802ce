// fwd_moments.cu -- key moments for the null floor of causal prefill (sm_100a).
//
// The null floor of a row ("Polar Attention: A Three-Channel Decomposition",
// ATMA technical summary, section 2.1) needs the mean and the population
// standard deviation of the row's visible logits, i.e. the two raw sums
//   S1_i = sum_{j<=i} <q_i,k_j> = <q_i, sum_j k_j>
//   S2_i = sum_{j<=i} <q_i,k_j>^2 = q_i^T (sum_j k_j k_j^T) q_i.
// Both are linear in the key moments sum_j k_j and sum_j k_j k_j^T, so for the
// keys of the full key tiles left of a query tile they can be taken from those
// moments once per row instead of once per (row, key).  This pre-pass writes,
// for every (batch, kv head) and every 128-key tile t that is full (t < the
// number of query tiles - 1), the moments of the keys from the start of t's
// chunk of kMomChunk tiles up to and including tile t:
//   rec[t][d*64 + e] = sum k_d k_e   (4096 fp32, a symmetric 64 x 64 Gram)
//   rec[t][4096 + d] = sum k_d       (64 fp32)
// The prefill kernel adds the records that close each earlier chunk to the
// record of its own last full tile, which gives the moments of all keys left of
// its query tile.
//
// One CTA per (chunk, batch x kv head), 8 warps.  A chunk's tiles stream
// through a two-buffer cp.async ring into padded shared rows (144 bytes, so the
// transposing ldmatrix reads are bank-conflict free); the Gram accumulates on
// the tensor cores (mma.sync m16n8k16, bf16 in, fp32 accumulate; the products
// of bf16 values are exact in fp32), warp w owning rows d in [16(w/2), +16) and
// columns e in [32(w%2), +32).  The accumulators carry across the chunk's
// tiles, so each record is an inclusive running sum.
#include "polar_common.cuh"
#include "polar_internal.h"

namespace polar {
namespace {

constexpr int kRowPitch = 144;                 // bytes per padded key row (64 bf16 + 16)
constexpr int kBufBytes = 128 * kRowPitch;     // one key tile

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                          uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__global__ void __launch_bounds__(256)
fwd_moments_kernel(const __nv_bfloat16 *__restrict__ k, float *__restrict__ rec, int T, int Hkv,
                   int nrec, int chunk0) {
    __shared__ __align__(128) uint8_t buf[2][kBufBytes];
    __shared__ float ks_part[4][kHeadDim];

    const int chunk = chunk0 + static_cast<int>(blockIdx.x), bg = blockIdx.y;  // bg = b * Hkv + g
    const int b = bg / Hkv, g = bg % Hkv;
    const int t_begin = chunk * kMomChunk;
    const int t_end = min(t_begin + kMomChunk, nrec);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    // Tile t's 128 key rows, 16-byte pieces: thread tid copies pieces tid + 256 i.
    auto load_tile = [&](int t, int slot) {
        const uint32_t base = smem_u32(buf[slot]);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int piece = tid + 256 * i;
            const int r = piece >> 3, c = piece & 7;
            const size_t key = static_cast<size_t>(t) * 128 + r;
            const __nv_bfloat16 *src =
                k + ((static_cast<size_t>(b) * T + key) * Hkv + g) * kHeadDim + 8 * c;
            cp_async16(base + r * kRowPitch + 16 * c, src);
        }
        cp_async_commit();
    };

    const int mt = warp >> 1;        // Gram rows d in [16 mt, 16 mt + 16)
    const int nb = 4 * (warp & 1);   // Gram column tiles nb .. nb+3 (8 columns each)
    float acc[4][4];
#pragma unroll
    for (int n = 0; n < 4; ++n)
#pragma unroll
        for (int x = 0; x < 4; ++x) acc[n][x] = 0.f;
    const int kd = tid & 63, kpart = tid >> 6;  // key-sum column and key quarter
    float ksum = 0.f;

    if (t_begin < t_end) load_tile(t_begin, 0);
    for (int t = t_begin; t < t_end; ++t) {
        const int slot = (t - t_begin) & 1;
        if (t + 1 < t_end) {
            load_tile(t + 1, slot ^ 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        const uint32_t base = smem_u32(buf[slot]);
        const int mi = lane >> 3, r8 = lane & 7;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            // A = K^T (rows d, columns keys): matrices (keys +0/+8) x (d +0/+8).
            uint32_t a[4];
            ldsm_x4_trans(base + (16 * ks + r8 + 8 * (mi >> 1)) * kRowPitch +
                              2 * (16 * mt + 8 * (mi & 1)),
                          a);
            // B = K (rows keys, columns e): per x4, two column tiles x (keys +0/+8).
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint32_t bb[4];
                ldsm_x4_trans(base + (16 * ks + r8 + 8 * (mi & 1)) * kRowPitch +
                                  2 * 8 * (nb + 2 * h + (mi >> 1)),
                              bb);
                mma_16816(acc[2 * h], a, bb[0], bb[1]);
                mma_16816(acc[2 * h + 1], a, bb[2], bb[3]);
            }
        }
        const __nv_bfloat16 *krow = reinterpret_cast<const __nv_bfloat16 *>(buf[slot]);
#pragma unroll 8
        for (int r = 32 * kpart; r < 32 * kpart + 32; ++r)
            ksum += __bfloat162float(krow[r * (kRowPitch / 2) + kd]);
        ks_part[kpart][kd] = ksum;
        __syncthreads();  // every read of buf[slot] and every ks_part write is done

        float *out = rec + (static_cast<size_t>(bg) * nrec + t) * kMomFloats;
        const int gr = lane >> 2, gc = 2 * (lane & 3);
#pragma unroll
        for (int n = 0; n < 4; ++n) {
            const int d = 16 * mt + gr, e = 8 * (nb + n) + gc;
            *reinterpret_cast<float2 *>(out + d * kHeadDim + e) = make_float2(acc[n][0], acc[n][1]);
            *reinterpret_cast<float2 *>(out + (d + 8) * kHeadDim + e) =
                make_float2(acc[n][2], acc[n][3]);
        }
        if (tid < kHeadDim)
            out[kHeadDim * kHeadDim + tid] =
                (ks_part[0][tid] + ks_part[1][tid]) + (ks_part[2][tid] + ks_part[3][tid]);
    }
}

}  // namespace

int fwd_moment_records(int T) {
    const int nqt = (T + 127) / 128;
    return nqt > 1 ? nqt - 1 : 0;
}

size_t fwd_moments_bytes(int B, int T, int Hkv) {
    return static_cast<size_t>(B) * Hkv * fwd_moment_records(T) * kMomFloats * sizeof(float);
}

cudaError_t launch_fwd_moments(const void *k, int B, int T, int Hkv, float *rec, int rec_lo,
                               int rec_hi, cudaStream_t stream) {
    const int nrec = fwd_moment_records(T);
    if (nrec == 0 || B == 0) return cudaSuccess;
    // Whole chunks: every record of a chunk is a running sum from the chunk's start.
    const int c_lo = max(rec_lo, 0) / kMomChunk;
    const int c_hi = (min(rec_hi, nrec) + kMomChunk - 1) / kMomChunk;
    if (c_hi <= c_lo) return cudaSuccess;
    const long long bg = static_cast<long long>(B) * Hkv;
    if (bg > 65535) return cudaErrorInvalidValue;
    fwd_moments_kernel<<<dim3(c_hi - c_lo, static_cast<unsigned>(bg)), 256, 0, stream>>>(
        static_cast<const __nv_bfloat16 *>(k), rec, T, Hkv, nrec, c_lo);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace polar
