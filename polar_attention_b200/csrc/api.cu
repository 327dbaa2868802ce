// api.cu -- the C ABI declared in include/polar_attn.h: argument validation,
// the per-device status word, tensor-map encoding and dispatch to the kernels.
#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>

#include <cudaTypedefs.h>

#include "polar_attn_selftest.h"
#include "polar_common.cuh"
#include "polar_gdelta.h"
#include "polar_internal.h"

namespace polar {

__device__ int g_status = 0;  // first device-side error since the last polar_attn_get_status

namespace {

std::atomic<uint64_t> g_launches{0};
std::mutex g_mu;
constexpr int kMaxDevices = 64;
int *g_status_addr[kMaxDevices] = {nullptr};
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

// Device address of g_status on the current device (looked up once per device).
int *status_ptr() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_status_addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_status) != cudaSuccess) return nullptr;
        g_status_addr[dev] = static_cast<int *>(p);
    }
    return g_status_addr[dev];
}

// Copy streams and events of the host-buffer prefill, created once per device:
// inputs go in on `in`, outputs come back on `out` (two copy engines), and a
// second compute stream `comp2` lets consecutive row segments' prefills
// overlap; all are joined to the caller's stream through events.  `mu`
// serialises host-buffer calls on a device, which share these.
struct HostPipe {
    std::mutex mu;
    bool ready = false;
    cudaStream_t in = nullptr, out = nullptr, comp2 = nullptr;
    cudaEvent_t start = nullptr, out_done = nullptr, kv_in = nullptr, mom_done = nullptr,
                comp2_done = nullptr, in_done[2] = {}, comp_done[2] = {};
};
HostPipe g_pipe[kMaxDevices];

HostPipe *host_pipe() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    HostPipe &hp = g_pipe[dev];
    std::lock_guard<std::mutex> lk(g_mu);
    if (!hp.ready) {
        const unsigned ef = cudaEventDisableTiming;
        if (cudaStreamCreateWithFlags(&hp.in, cudaStreamNonBlocking) != cudaSuccess ||
            cudaStreamCreateWithFlags(&hp.out, cudaStreamNonBlocking) != cudaSuccess ||
            cudaStreamCreateWithFlags(&hp.comp2, cudaStreamNonBlocking) != cudaSuccess ||
            cudaEventCreateWithFlags(&hp.start, ef) != cudaSuccess ||
            cudaEventCreateWithFlags(&hp.out_done, ef) != cudaSuccess ||
            cudaEventCreateWithFlags(&hp.kv_in, ef) != cudaSuccess ||
            cudaEventCreateWithFlags(&hp.mom_done, ef) != cudaSuccess ||
            cudaEventCreateWithFlags(&hp.comp2_done, ef) != cudaSuccess)
            return nullptr;
        for (int i = 0; i < 2; ++i)
            if (cudaEventCreateWithFlags(&hp.in_done[i], ef) != cudaSuccess ||
                cudaEventCreateWithFlags(&hp.comp_done[i], ef) != cudaSuccess)
                return nullptr;
        hp.ready = true;
    }
    return &hp;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

size_t dtype_bytes(int dtype) { return dtype == POLAR_FP32 ? 4 : 2; }

polar_status_t check_common(const polar_params_t *p) {
    if (!p) return POLAR_ERR_INVALID_ARG;
    if (p->head_dim != kHeadDim) return POLAR_ERR_UNSUPPORTED;
    if (p->Hq <= 0 || p->Hkv <= 0 || p->Hq % p->Hkv != 0) return POLAR_ERR_INVALID_ARG;
    if (p->dtype != POLAR_BF16 && p->dtype != POLAR_FP32) return POLAR_ERR_INVALID_ARG;
    if (!(p->logit_scale > 0.0f) || !std::isfinite(p->logit_scale)) return POLAR_ERR_INVALID_ARG;
    if (!(p->alpha >= 0.0f) || !std::isfinite(p->alpha)) return POLAR_ERR_INVALID_ARG;
    if (!std::isfinite(p->beta)) return POLAR_ERR_INVALID_ARG;
    if (p->L_train < 2) return POLAR_ERR_INVALID_ARG;
    if (p->window < 0) return POLAR_ERR_INVALID_ARG;
    return POLAR_OK;
}

polar_status_t check_fwd(const polar_params_t *p) {
    polar_status_t st = check_common(p);
    if (st != POLAR_OK) return st;
    if (p->B < 0 || p->T < 0) return POLAR_ERR_INVALID_ARG;
    if (p->causal != 1) return POLAR_ERR_UNSUPPORTED;
    if (p->impl < POLAR_IMPL_AUTO || p->impl > POLAR_IMPL_TC) return POLAR_ERR_INVALID_ARG;
    if (p->T > (1 << 30) / 64 || p->B > 65535 || p->Hq > 65535) return POLAR_ERR_UNSUPPORTED;
    return POLAR_OK;
}

polar_status_t check_decode(const polar_params_t *p, int num_seqs, int max_pages) {
    polar_status_t st = check_common(p);
    if (st != POLAR_OK) return st;
    if (p->dtype != POLAR_BF16) return POLAR_ERR_UNSUPPORTED;
    const int G = p->Hq / p->Hkv;
    if (G != 1 && G != 2 && G != 4 && G != 8) return POLAR_ERR_UNSUPPORTED;
    if (num_seqs < 0 || num_seqs > 65535 || max_pages < 1) return POLAR_ERR_INVALID_ARG;
    if (static_cast<long long>(max_pages) * kPage > (1ll << 31) - 1) return POLAR_ERR_INVALID_ARG;
    return POLAR_OK;
}

// Multi-token decode: every row of the mma tile is a (chunk token, query head)
// pair of one kv group, so G * chunk rows must fit the 16 of one tile; the
// merge grid's second dimension is num_seqs * chunk.
polar_status_t check_decode_chunk(const polar_params_t *p, int num_seqs, int max_pages, int chunk) {
    polar_status_t st = check_decode(p, num_seqs, max_pages);
    if (st != POLAR_OK) return st;
    if (chunk < 1) return POLAR_ERR_INVALID_ARG;
    if ((p->Hq / p->Hkv) * chunk > 16) return POLAR_ERR_UNSUPPORTED;
    if (static_cast<long long>(num_seqs) * chunk > 65535) return POLAR_ERR_UNSUPPORTED;
    return POLAR_OK;
}

// Memory channel: shape and flag checks shared by prefill and step.
polar_status_t check_gdelta(const polar_gdelta_params_t *p) {
    if (!p) return POLAR_ERR_INVALID_ARG;
    if (p->head_dim != kHeadDim) return POLAR_ERR_UNSUPPORTED;
    if (p->dtype != POLAR_BF16 && p->dtype != POLAR_FP32) return POLAR_ERR_INVALID_ARG;
    if (p->H <= 0) return POLAR_ERR_INVALID_ARG;
    if ((p->zero_init != 0 && p->zero_init != 1) || (p->accumulate != 0 && p->accumulate != 1))
        return POLAR_ERR_INVALID_ARG;
    return POLAR_OK;
}

// Prefill: the scan grid's second dimension is B * H.
polar_status_t check_gdelta_prefill(const polar_gdelta_params_t *p) {
    polar_status_t st = check_gdelta(p);
    if (st != POLAR_OK) return st;
    if (p->B < 0 || p->T < 0) return POLAR_ERR_INVALID_ARG;
    if (static_cast<long long>(p->B) * p->H > 65535) return POLAR_ERR_UNSUPPORTED;
    return POLAR_OK;
}

bool aligned4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

polar_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? POLAR_OK : POLAR_ERR_CUDA; }

FwdLaunch make_fwd(const void *q, const void *k, const void *v, const float *u,
                   const polar_params_t *p, void *out, float *neff, int *status,
                   cudaStream_t stream) {
    FwdLaunch a;
    a.q = q; a.k = k; a.v = v; a.u = u; a.out = out; a.neff = neff;
    a.B = p->B; a.T = p->T; a.Hq = p->Hq; a.Hkv = p->Hkv; a.dtype = p->dtype;
    a.s = p->logit_scale; a.alpha = p->alpha; a.beta = p->beta; a.L = p->L_train;
    a.window = p->window;
    a.status = status; a.moments = nullptr; a.state = nullptr; a.stream = stream;
    a.qt_lo = 0; a.qt_cnt = 0; a.moments_ready = false;
    return a;
}

}  // namespace

void count_launches(int n) { g_launches.fetch_add(static_cast<uint64_t>(n)); }

int *device_status_word() { return status_ptr(); }

// One bounded wait on a barrier that no thread or copy ever completes.
__global__ void selftest_timeout_kernel(int *status) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait(&bar, 0, status);
}

CUresult encode_tiled(CUtensorMap *map, CUtensorMapDataType dtype, uint32_t rank, void *base,
                      const uint64_t *dims, const uint64_t *strides_bytes, const uint32_t *box,
                      CUtensorMapSwizzle swizzle) {
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (!g_encode) {
            void *fn = nullptr;
            cudaDriverEntryPointQueryResult q;
            if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
                    cudaSuccess ||
                q != cudaDriverEntryPointSuccess || !fn)
                return CUDA_ERROR_NOT_FOUND;
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
        }
    }
    uint32_t estr[5] = {1, 1, 1, 1, 1};
    return g_encode(map, dtype, rank, base, dims, strides_bytes, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

}  // namespace polar

using namespace polar;

extern "C" {

void polar_attn_default_params(polar_params_t *p, int B, int T, int Hq, int Hkv, int dtype) {
    if (!p) return;
    std::memset(p, 0, sizeof *p);
    p->B = B; p->T = T; p->Hq = Hq; p->Hkv = Hkv; p->head_dim = kHeadDim; p->dtype = dtype;
    p->logit_scale = 8.0f; p->alpha = 0.3f; p->L_train = 2048; p->beta = 1.0f;
    p->causal = 1; p->impl = POLAR_IMPL_AUTO;
}

size_t polar_attn_fwd_workspace_size(const polar_params_t *p) {
    if (check_fwd(p) != POLAR_OK) return 0;
    return fwd_moments_bytes(p->B, p->T, p->Hkv);
}

polar_status_t polar_attn_fwd(const void *q, const void *k, const void *v, const float *u,
                              const polar_params_t *params, void *out, float *neff_out,
                              void *stream) {
    return polar_attn_fwd_ws(q, k, v, u, params, out, neff_out, nullptr, 0, stream);
}

polar_status_t polar_attn_fwd_ws(const void *q, const void *k, const void *v, const float *u,
                                 const polar_params_t *params, void *out, float *neff_out,
                                 void *workspace, size_t ws_bytes, void *stream) {
    polar_status_t st = check_fwd(params);
    if (st != POLAR_OK) return st;
    if (params->B == 0 || params->T == 0) return POLAR_OK;
    if (!q || !k || !v || !u || !out) return POLAR_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(u) || !aligned16(out) ||
        (neff_out && (reinterpret_cast<uintptr_t>(neff_out) & 3u)) ||
        (workspace && !aligned16(workspace)))
        return POLAR_ERR_INVALID_ARG;
    if (workspace && ws_bytes < fwd_moments_bytes(params->B, params->T, params->Hkv))
        return POLAR_ERR_WORKSPACE;
    int *status = status_ptr();
    if (!status) return POLAR_ERR_CUDA;
    FwdLaunch a = make_fwd(q, k, v, u, params, out, neff_out, status,
                           static_cast<cudaStream_t>(stream));
    // Key moments beyond one tile; the tensor-core launcher decides where they
    // pay off (enough query tiles, or a long enough window).
    a.moments = fwd_moment_records(params->T) > 0 ? static_cast<float *>(workspace) : nullptr;
    // The tensor-core kernel pairs two query heads of one key/value group per
    // CTA, so it needs an even group size; fp32 inputs use the CUDA-core kernel.
    const bool tc_ok = params->dtype == POLAR_BF16 && (params->Hq / params->Hkv) % 2 == 0;
    const bool tc = params->impl == POLAR_IMPL_TC || (params->impl == POLAR_IMPL_AUTO && tc_ok);
    if (tc) {
        if (!tc_ok) return POLAR_ERR_UNSUPPORTED;
        return from_cuda(launch_fwd_tc(a));
    }
    return from_cuda(launch_fwd_simt(a));
}

size_t polar_attn_bwd_workspace_size(const polar_params_t *p) {
    if (check_fwd(p) != POLAR_OK) return 0;
    return bwd_workspace_bytes(p->B, p->T, p->Hq);
}

polar_status_t polar_attn_bwd(const void *q, const void *k, const void *v, const float *u,
                              const void *dout, const polar_params_t *p, float *dq, float *dk,
                              float *dv, float *du, void *workspace, size_t ws_bytes,
                              void *stream) {
    polar_status_t st = check_fwd(p);
    if (st != POLAR_OK) return st;
    if (!du || !aligned16(du)) return POLAR_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (p->B == 0 || p->T == 0)
        return from_cuda(cudaMemsetAsync(du, 0, static_cast<size_t>(p->Hq) * kHeadDim * 4, s));
    if (!q || !k || !v || !u || !dout || !dq || !dk || !dv || !workspace)
        return POLAR_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(u) || !aligned16(dout) ||
        !aligned16(dq) || !aligned16(dk) || !aligned16(dv) || !aligned16(workspace))
        return POLAR_ERR_INVALID_ARG;
    if (ws_bytes < bwd_workspace_bytes(p->B, p->T, p->Hq)) return POLAR_ERR_WORKSPACE;
    int *status = status_ptr();
    if (!status) return POLAR_ERR_CUDA;
    BwdLaunch a;
    a.q = q; a.k = k; a.v = v; a.dout = dout; a.u = u;
    a.dq = dq; a.dk = dk; a.dv = dv; a.du = du;
    a.B = p->B; a.T = p->T; a.Hq = p->Hq; a.Hkv = p->Hkv; a.dtype = p->dtype;
    a.s = p->logit_scale; a.alpha = p->alpha; a.beta = p->beta; a.L = p->L_train;
    a.window = p->window; a.workspace = workspace; a.status = status; a.stream = s;
    return from_cuda(launch_bwd(a));
}

size_t polar_attn_fwd_state_size(const polar_params_t *p) {
    if (check_fwd(p) != POLAR_OK) return 0;
    return static_cast<size_t>(p->B) * p->Hq * p->T * kFwdStateWords * sizeof(float);
}

polar_status_t polar_attn_fwd_train(const void *q, const void *k, const void *v, const float *u,
                                    const polar_params_t *params, void *out, float *neff_out,
                                    float *state, void *stream) {
    polar_status_t st = check_fwd(params);
    if (st != POLAR_OK) return st;
    if (params->B == 0 || params->T == 0) return POLAR_OK;
    if (!state || !aligned16(state)) return POLAR_ERR_INVALID_ARG;
    const int sup = fwd_state_supported(params->dtype, params->T, params->Hq, params->Hkv,
                                        params->logit_scale, params->alpha, params->L_train,
                                        params->window);
    if (sup < 0) return POLAR_ERR_CUDA;
    // No saved state for this shape: the plain forward (the backward then
    // recomputes the rows).
    if (sup == 0 || params->impl == POLAR_IMPL_SIMT)
        return polar_attn_fwd_ws(q, k, v, u, params, out, neff_out, nullptr, 0, stream);
    if (!q || !k || !v || !u || !out) return POLAR_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(u) || !aligned16(out) ||
        (neff_out && (reinterpret_cast<uintptr_t>(neff_out) & 3u)))
        return POLAR_ERR_INVALID_ARG;
    int *status = status_ptr();
    if (!status) return POLAR_ERR_CUDA;
    FwdLaunch a = make_fwd(q, k, v, u, params, out, neff_out, status,
                           static_cast<cudaStream_t>(stream));
    a.state = state;
    return from_cuda(launch_fwd_train_tc(a));
}

polar_status_t polar_attn_bwd_from_state(const void *q, const void *k, const void *v,
                                         const float *u, const void *out, const float *state,
                                         const void *dout, const polar_params_t *p, float *dq,
                                         float *dk, float *dv, float *du, void *workspace,
                                         size_t ws_bytes, void *stream) {
    polar_status_t st = check_fwd(p);
    if (st != POLAR_OK) return st;
    if (!du || !aligned16(du)) return POLAR_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (p->B == 0 || p->T == 0)
        return from_cuda(cudaMemsetAsync(du, 0, static_cast<size_t>(p->Hq) * kHeadDim * 4, s));
    if (!q || !k || !v || !u || !out || !state || !dout || !dq || !dk || !dv || !workspace)
        return POLAR_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(u) || !aligned16(out) ||
        !aligned16(state) || !aligned16(dout) || !aligned16(dq) || !aligned16(dk) ||
        !aligned16(dv) || !aligned16(workspace))
        return POLAR_ERR_INVALID_ARG;
    if (ws_bytes < bwd_workspace_bytes(p->B, p->T, p->Hq)) return POLAR_ERR_WORKSPACE;
    int *status = status_ptr();
    if (!status) return POLAR_ERR_CUDA;
    BwdLaunch a;
    a.q = q; a.k = k; a.v = v; a.dout = dout; a.u = u;
    a.dq = dq; a.dk = dk; a.dv = dv; a.du = du;
    a.B = p->B; a.T = p->T; a.Hq = p->Hq; a.Hkv = p->Hkv; a.dtype = p->dtype;
    a.s = p->logit_scale; a.alpha = p->alpha; a.beta = p->beta; a.L = p->L_train;
    a.window = p->window; a.workspace = workspace; a.status = status; a.stream = s;
    if (p->impl == POLAR_IMPL_SIMT) return from_cuda(launch_bwd(a));
    return from_cuda(launch_bwd_from_state(a, out, state));
}

namespace {

// Row segments of a host-buffer tensor-core prefill of T rows, from the last
// rows to the first: about T/4 rows from the top, then halves down to 1024
// rows (one segment below T = 2048).  Boundaries fall on 128-row query tiles.
// Writes at most `cap` segments (the last one always ends at row 0) and
// returns how many.
int fwd_host_segments(int T, int *seg_lo, int *seg_hi, int cap) {
    const int seg = T >= 2048 ? static_cast<int>(round_up((T + 3) / 4, 128)) : T;
    int n = 0;
    for (int hi = T, lo = 0; hi > 0 && n < cap; hi = lo, ++n) {
        lo = seg == T ? 0
             : hi > seg  ? static_cast<int>(round_up(static_cast<size_t>(hi - seg), 128))
             : hi > 1024 ? hi / 2 / 128 * 128
                         : 0;
        if (n == cap - 1) lo = 0;
        seg_lo[n] = lo;
        seg_hi[n] = hi;
    }
    return n;
}

}  // namespace

int polar_attn_selftest_fwd_host_segments(int T, int *seg_lo, int *seg_hi, int cap) {
    if (T < 0 || cap < 1 || !seg_lo || !seg_hi) return -1;
    return fwd_host_segments(T, seg_lo, seg_hi, cap);
}

size_t polar_attn_fwd_staging_size(const polar_params_t *p) {
    if (check_fwd(p) != POLAR_OK) return 0;
    const size_t e = dtype_bytes(p->dtype);
    const size_t rows = static_cast<size_t>(p->B) * p->T;
    size_t n = 0;
    n += round_up(rows * p->Hq * kHeadDim * e, 256);       // q
    n += 2 * round_up(rows * p->Hkv * kHeadDim * e, 256);  // k, v
    n += round_up(static_cast<size_t>(p->Hq) * kHeadDim * 4, 256);  // u
    n += round_up(rows * p->Hq * kHeadDim * e, 256);       // out
    n += round_up(rows * p->Hq * 4, 256);                  // neff
    n += round_up(fwd_moments_bytes(p->B, p->T, p->Hkv), 256);  // workspace
    return n;
}

polar_status_t polar_attn_fwd_host(const void *q_h, const void *k_h, const void *v_h,
                                   const float *u_h, const polar_params_t *p, void *out_h,
                                   float *neff_h, void *staging, size_t staging_bytes,
                                   void *stream) {
    polar_status_t st = check_fwd(p);
    if (st != POLAR_OK) return st;
    if (p->B == 0 || p->T == 0) return POLAR_OK;
    if (!q_h || !k_h || !v_h || !u_h || !out_h || !staging) return POLAR_ERR_INVALID_ARG;
    if (staging_bytes < polar_attn_fwd_staging_size(p)) return POLAR_ERR_WORKSPACE;
    if (!aligned16(staging)) return POLAR_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t e = dtype_bytes(p->dtype);
    const size_t rows = static_cast<size_t>(p->B) * p->T;
    const size_t qb = rows * p->Hq * kHeadDim * e, kb = rows * p->Hkv * kHeadDim * e;
    const size_t ub = static_cast<size_t>(p->Hq) * kHeadDim * 4, nb = rows * p->Hq * 4;
    char *base = static_cast<char *>(staging);
    char *dq = base;
    char *dk = dq + round_up(qb, 256);
    char *dv = dk + round_up(kb, 256);
    char *du = dv + round_up(kb, 256);
    char *dout = du + round_up(ub, 256);
    char *dne = dout + round_up(qb, 256);
    char *dws = dne + round_up(nb, 256);
    HostPipe *hp = host_pipe();
    if (!hp) return POLAR_ERR_CUDA;
    std::lock_guard<std::mutex> lk(hp->mu);
    const size_t qbb = qb / p->B, kbb = kb / p->B, nbb = nb / p->B;  // one batch
    polar_params_t p1 = *p;
    p1.B = 1;
    const size_t wsb = fwd_moments_bytes(1, p->T, p->Hkv);
    const char *qh = static_cast<const char *>(q_h), *kh = static_cast<const char *>(k_h),
               *vh = static_cast<const char *>(v_h);
    char *oh = static_cast<char *>(out_h), *nh = reinterpret_cast<char *>(neff_h);
    // The copies and the second compute stream start after earlier work on
    // `stream` (which may still use the staging).
    if (cudaEventRecord(hp->start, s) != cudaSuccess ||
        cudaStreamWaitEvent(hp->in, hp->start, 0) != cudaSuccess ||
        cudaStreamWaitEvent(hp->out, hp->start, 0) != cudaSuccess ||
        cudaStreamWaitEvent(hp->comp2, hp->start, 0) != cudaSuccess ||
        cudaMemcpyAsync(du, u_h, ub, cudaMemcpyHostToDevice, hp->in) != cudaSuccess)
        return POLAR_ERR_CUDA;
    const bool tc = p->dtype == POLAR_BF16 && (p->Hq / p->Hkv) % 2 == 0 && p->impl != POLAR_IMPL_SIMT;
    const size_t qrow = static_cast<size_t>(p->Hq) * kHeadDim * e, krow = static_cast<size_t>(p->Hkv) * kHeadDim * e;
    int *status = status_ptr();
    if (!status) return POLAR_ERR_CUDA;
    // Copies rows lo .. hi - 1 of batch b's output back once `done` (recorded on
    // the stream that computed them) has passed.
    auto send_back = [&](int b, int lo, int hi, cudaEvent_t done) {
        const size_t rows_s = static_cast<size_t>(hi - lo);
        const size_t qo = b * qbb + lo * qrow;
        return cudaStreamWaitEvent(hp->out, done, 0) == cudaSuccess &&
               cudaMemcpyAsync(oh + qo, dout + qo, rows_s * qrow, cudaMemcpyDeviceToHost, hp->out) ==
                   cudaSuccess;
    };
    // Batch b's n_eff ([Hq, T], contiguous) in one copy, queued on the output
    // stream after the copies of all its segments, which waited for each of
    // their prefills: one 2-D copy per segment (Hq strided runs) costs the
    // output stream far more than the bytes.
    auto send_neff = [&](int b) {
        return !neff_h || cudaMemcpyAsync(nh + b * nbb, dne + b * nbb, nbb, cudaMemcpyDeviceToHost,
                                          hp->out) == cudaSuccess;
    };
    if (!tc) {
        // CUDA-core prefill: whole batches; the inputs of batch b+1 go in and
        // the outputs of batch b-1 come back while batch b runs.
        for (int b = 0; b < p->B; ++b) {
            const int e2 = b & 1;
            if (cudaMemcpyAsync(dq + b * qbb, qh + b * qbb, qbb, cudaMemcpyHostToDevice, hp->in) != cudaSuccess ||
                cudaMemcpyAsync(dk + b * kbb, kh + b * kbb, kbb, cudaMemcpyHostToDevice, hp->in) != cudaSuccess ||
                cudaMemcpyAsync(dv + b * kbb, vh + b * kbb, kbb, cudaMemcpyHostToDevice, hp->in) != cudaSuccess ||
                cudaEventRecord(hp->in_done[e2], hp->in) != cudaSuccess ||
                cudaStreamWaitEvent(s, hp->in_done[e2], 0) != cudaSuccess)
                return POLAR_ERR_CUDA;
            float *ne = neff_h ? reinterpret_cast<float *>(dne + b * nbb) : nullptr;
            st = polar_attn_fwd_ws(dq + b * qbb, dk + b * kbb, dv + b * kbb, reinterpret_cast<float *>(du),
                                   &p1, dout + b * qbb, ne, wsb ? dws : nullptr, wsb, stream);
            if (st != POLAR_OK) return st;
            if (cudaEventRecord(hp->comp_done[e2], s) != cudaSuccess ||
                !send_back(b, 0, p->T, hp->comp_done[e2]) || !send_neff(b))
                return POLAR_ERR_CUDA;
        }
    } else {
        // Tensor-core prefill, batch by batch.  A batch's keys and values go in
        // first and its key moments are formed; then its queries go in row
        // segment by row segment from the LAST rows to the first.  A segment's
        // prefill then needs nothing that is still in flight but its own
        // queries, so the heaviest segments (the longest causal rows) start
        // first and the call ends on the lightest one, whose output copy is
        // short.  Segments alternate between `stream` and a second compute
        // stream, so that a segment's prefill fills the SMs that the previous
        // one's last wave leaves idle; every segment's outputs go back as soon
        // as it is done (segments: fwd_host_segments).
        const int nqt = (p->T + 127) / 128;
        constexpr int kMaxSeg = 64;
        int seg_lo[kMaxSeg], seg_hi[kMaxSeg];
        const int nseg = fwd_host_segments(p->T, seg_lo, seg_hi, kMaxSeg);
        int ev = 0;
        for (int b = 0; b < p->B; ++b) {
            if (cudaMemcpyAsync(dk + b * kbb, kh + b * kbb, kbb, cudaMemcpyHostToDevice, hp->in) != cudaSuccess ||
                cudaMemcpyAsync(dv + b * kbb, vh + b * kbb, kbb, cudaMemcpyHostToDevice, hp->in) != cudaSuccess ||
                cudaEventRecord(hp->kv_in, hp->in) != cudaSuccess ||
                cudaStreamWaitEvent(s, hp->kv_in, 0) != cudaSuccess)
                return POLAR_ERR_CUDA;
            float *ne = neff_h ? reinterpret_cast<float *>(dne + b * nbb) : nullptr;
            FwdLaunch a = make_fwd(dq + b * qbb, dk + b * kbb, dv + b * kbb, reinterpret_cast<float *>(du),
                                   &p1, dout + b * qbb, ne, status, s);
            a.moments = wsb ? reinterpret_cast<float *>(dws + b * wsb) : nullptr;
            if (fwd_tc_reads_moments(a) &&
                launch_fwd_moments(a.k, 1, p->T, p->Hkv, a.moments, 0, nqt - 1, s) != cudaSuccess)
                return POLAR_ERR_CUDA;
            a.moments_ready = true;
            if (cudaEventRecord(hp->mom_done, s) != cudaSuccess ||
                cudaStreamWaitEvent(hp->comp2, hp->mom_done, 0) != cudaSuccess)
                return POLAR_ERR_CUDA;
            for (int k = 0; k < nseg; ++k, ++ev) {
                const int lo = seg_lo[k], hi = seg_hi[k];
                const int e2 = ev & 1;
                cudaStream_t cs = e2 ? hp->comp2 : s;
                const size_t qo = b * qbb + lo * qrow;
                if (cudaMemcpyAsync(dq + qo, qh + qo, static_cast<size_t>(hi - lo) * qrow,
                                    cudaMemcpyHostToDevice, hp->in) != cudaSuccess ||
                    cudaEventRecord(hp->in_done[e2], hp->in) != cudaSuccess ||
                    cudaStreamWaitEvent(cs, hp->in_done[e2], 0) != cudaSuccess)
                    return POLAR_ERR_CUDA;
                a.stream = cs;
                a.qt_lo = lo / 128;
                a.qt_cnt = (hi + 127) / 128 - a.qt_lo;
                st = from_cuda(launch_fwd_tc(a));
                if (st != POLAR_OK) return st;
                if (cudaEventRecord(hp->comp_done[e2], cs) != cudaSuccess ||
                    !send_back(b, lo, hi, hp->comp_done[e2]))
                    return POLAR_ERR_CUDA;
            }
            if (!send_neff(b)) return POLAR_ERR_CUDA;
        }
        if (cudaEventRecord(hp->comp2_done, hp->comp2) != cudaSuccess ||
            cudaStreamWaitEvent(s, hp->comp2_done, 0) != cudaSuccess)
            return POLAR_ERR_CUDA;
    }
    if (cudaEventRecord(hp->out_done, hp->out) != cudaSuccess ||
        cudaStreamWaitEvent(s, hp->out_done, 0) != cudaSuccess)
        return POLAR_ERR_CUDA;
    return from_cuda(cudaStreamSynchronize(s));
}

size_t polar_attn_decode_workspace_size(int num_seqs, int max_pages, const polar_params_t *p) {
    if (check_decode(p, num_seqs, max_pages) != POLAR_OK) return 0;
    return decode_partials_bytes(num_seqs, max_pages, p->Hq, p->Hkv, 1);
}

size_t polar_attn_decode_chunk_workspace_size(int num_seqs, int max_pages, int chunk,
                                              const polar_params_t *p) {
    if (check_decode_chunk(p, num_seqs, max_pages, chunk) != POLAR_OK) return 0;
    return decode_partials_bytes(num_seqs, max_pages, p->Hq, p->Hkv, chunk);
}

polar_status_t polar_attn_decode_paged(const void *q, const void *kv_pages, int num_pages,
                                       const int32_t *page_table, int max_pages,
                                       const int32_t *seqlens, int num_seqs, const float *u,
                                       const polar_params_t *p, void *out, float *neff_out,
                                       void *workspace, size_t ws_bytes, void *stream) {
    return polar_attn_decode_paged_chunk(q, kv_pages, num_pages, page_table, max_pages, seqlens,
                                         num_seqs, 1, u, p, out, neff_out, workspace, ws_bytes,
                                         stream);
}

polar_status_t polar_attn_decode_paged_chunk(const void *q, const void *kv_pages, int num_pages,
                                             const int32_t *page_table, int max_pages,
                                             const int32_t *seqlens, int num_seqs, int chunk,
                                             const float *u, const polar_params_t *p, void *out,
                                             float *neff_out, void *workspace, size_t ws_bytes,
                                             void *stream) {
    polar_status_t st = check_decode_chunk(p, num_seqs, max_pages, chunk);
    if (st != POLAR_OK) return st;
    if (num_seqs == 0) return POLAR_OK;
    if (num_pages < 1 || static_cast<long long>(num_pages) * 2 * p->Hkv * kPage > (1ll << 31) - 1)
        return POLAR_ERR_INVALID_ARG;
    if (!q || !kv_pages || !page_table || !seqlens || !u || !out || !workspace)
        return POLAR_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(kv_pages) || !aligned16(u) || !aligned16(out) ||
        !aligned16(workspace) || (reinterpret_cast<uintptr_t>(page_table) & 3u) ||
        (reinterpret_cast<uintptr_t>(seqlens) & 3u) ||
        (neff_out && (reinterpret_cast<uintptr_t>(neff_out) & 3u)))
        return POLAR_ERR_INVALID_ARG;
    if (ws_bytes < decode_partials_bytes(num_seqs, max_pages, p->Hq, p->Hkv, chunk))
        return POLAR_ERR_WORKSPACE;
    int *status = status_ptr();
    if (!status) return POLAR_ERR_CUDA;
    DecodeLaunch a;
    a.chunk = chunk;
    a.per_head = 0;
    a.q = q; a.kv_pages = kv_pages; a.num_pages = num_pages; a.page_table = page_table;
    a.max_pages = max_pages; a.seqlens = seqlens; a.num_seqs = num_seqs; a.u = u; a.out = out;
    a.neff = neff_out; a.Hq = p->Hq; a.Hkv = p->Hkv; a.s = p->logit_scale; a.alpha = p->alpha;
    a.beta = p->beta; a.L = p->L_train; a.window = p->window; a.workspace = workspace;
    a.status = status;
    a.stream = static_cast<cudaStream_t>(stream);
    return from_cuda(launch_decode(a));
}

size_t polar_attn_decode_staging_size(int num_seqs, int max_pages, const polar_params_t *p) {
    if (check_decode(p, num_seqs, max_pages) != POLAR_OK) return 0;
    const size_t e = dtype_bytes(p->dtype);
    size_t n = 0;
    n += round_up(static_cast<size_t>(num_seqs) * p->Hq * kHeadDim * e, 256);  // q
    n += round_up(static_cast<size_t>(num_seqs) * max_pages * 4, 256);         // page table
    n += round_up(static_cast<size_t>(num_seqs) * 4, 256);                     // seqlens
    n += round_up(static_cast<size_t>(p->Hq) * kHeadDim * 4, 256);             // u
    n += round_up(static_cast<size_t>(num_seqs) * p->Hq * kHeadDim * e, 256);  // out
    n += round_up(static_cast<size_t>(num_seqs) * p->Hq * 4, 256);             // neff
    n += round_up(decode_partials_bytes(num_seqs, max_pages, p->Hq, p->Hkv, 1), 256);
    return n;
}

polar_status_t polar_attn_decode_paged_host(const void *q_h, const void *kv_pages, int num_pages,
                                            const int32_t *page_table_h, int max_pages,
                                            const int32_t *seqlens_h, int num_seqs,
                                            const float *u_h, const polar_params_t *p,
                                            void *out_h, float *neff_h, void *staging,
                                            size_t staging_bytes, void *stream) {
    polar_status_t st = check_decode(p, num_seqs, max_pages);
    if (st != POLAR_OK) return st;
    if (num_seqs == 0) return POLAR_OK;
    if (!q_h || !page_table_h || !seqlens_h || !u_h || !out_h || !staging)
        return POLAR_ERR_INVALID_ARG;
    if (staging_bytes < polar_attn_decode_staging_size(num_seqs, max_pages, p))
        return POLAR_ERR_WORKSPACE;
    if (!aligned16(staging)) return POLAR_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t e = dtype_bytes(p->dtype);
    const size_t qb = static_cast<size_t>(num_seqs) * p->Hq * kHeadDim * e;
    const size_t ptb = static_cast<size_t>(num_seqs) * max_pages * 4;
    const size_t slb = static_cast<size_t>(num_seqs) * 4;
    const size_t ub = static_cast<size_t>(p->Hq) * kHeadDim * 4;
    const size_t nb = static_cast<size_t>(num_seqs) * p->Hq * 4;
    const size_t wsb = decode_partials_bytes(num_seqs, max_pages, p->Hq, p->Hkv, 1);
    char *dq = static_cast<char *>(staging);
    char *dpt = dq + round_up(qb, 256);
    char *dsl = dpt + round_up(ptb, 256);
    char *du = dsl + round_up(slb, 256);
    char *dout = du + round_up(ub, 256);
    char *dne = dout + round_up(qb, 256);
    char *dws = dne + round_up(nb, 256);
    if (cudaMemcpyAsync(dq, q_h, qb, cudaMemcpyHostToDevice, s) != cudaSuccess ||
        cudaMemcpyAsync(dpt, page_table_h, ptb, cudaMemcpyHostToDevice, s) != cudaSuccess ||
        cudaMemcpyAsync(dsl, seqlens_h, slb, cudaMemcpyHostToDevice, s) != cudaSuccess ||
        cudaMemcpyAsync(du, u_h, ub, cudaMemcpyHostToDevice, s) != cudaSuccess)
        return POLAR_ERR_CUDA;
    st = polar_attn_decode_paged(dq, kv_pages, num_pages, reinterpret_cast<int32_t *>(dpt),
                                 max_pages, reinterpret_cast<int32_t *>(dsl), num_seqs,
                                 reinterpret_cast<float *>(du), p, dout,
                                 neff_h ? reinterpret_cast<float *>(dne) : nullptr, dws, wsb,
                                 stream);
    if (st != POLAR_OK) return st;
    if (cudaMemcpyAsync(out_h, dout, qb, cudaMemcpyDeviceToHost, s) != cudaSuccess) return POLAR_ERR_CUDA;
    if (neff_h && cudaMemcpyAsync(neff_h, dne, nb, cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return POLAR_ERR_CUDA;
    return from_cuda(cudaStreamSynchronize(s));
}

polar_status_t polar_attn_get_status(void *stream) {
    int *status = status_ptr();
    if (!status) return POLAR_ERR_CUDA;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return POLAR_ERR_CUDA;
    int v = 0;
    if (cudaMemcpy(&v, status, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess) return POLAR_ERR_CUDA;
    const int zero = 0;
    if (cudaMemcpy(status, &zero, sizeof zero, cudaMemcpyHostToDevice) != cudaSuccess)
        return POLAR_ERR_CUDA;
    return static_cast<polar_status_t>(v);
}

const char *polar_attn_status_string(polar_status_t s) {
    switch (s) {
        case POLAR_OK: return "ok";
        case POLAR_ERR_INVALID_ARG: return "invalid argument, shape, stride or alignment";
        case POLAR_ERR_UNSUPPORTED: return "unsupported configuration";
        case POLAR_ERR_WORKSPACE: return "workspace or staging buffer too small";
        case POLAR_ERR_BAD_PAGE: return "page id outside the page pool";
        case POLAR_ERR_TIMEOUT: return "a bounded device wait timed out";
        case POLAR_ERR_CUDA: return "CUDA runtime error";
        case POLAR_ERR_BAD_SEQLEN: return "sequence length outside [1, 64*max_pages]";
        case POLAR_ERR_BAD_SLOT: return "memory state slot outside the state pool";
    }
    return "unknown status";
}

uint64_t polar_attn_launch_count(void) { return g_launches.load(); }

polar_status_t polar_attn_selftest_timeout(void *stream) {
    int *status = status_ptr();
    if (!status) return POLAR_ERR_CUDA;
    selftest_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(status);
    count_launches(1);
    return from_cuda(cudaGetLastError());
}

polar_status_t polar_attn_selftest_decode_per_head(const void *q, const void *kv_pages,
                                                   int num_pages, const int32_t *page_table,
                                                   int max_pages, const int32_t *seqlens,
                                                   int num_seqs, const float *u,
                                                   const polar_params_t *p, void *out,
                                                   float *neff_out, void *workspace,
                                                   size_t ws_bytes, void *stream) {
    polar_status_t st = check_decode(p, num_seqs, max_pages);
    if (st != POLAR_OK) return st;
    if (num_seqs == 0) return POLAR_OK;
    if (num_pages < 1 || static_cast<long long>(num_pages) * 2 * p->Hkv * kPage > (1ll << 31) - 1)
        return POLAR_ERR_INVALID_ARG;
    if (!q || !kv_pages || !page_table || !seqlens || !u || !out || !workspace)
        return POLAR_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(kv_pages) || !aligned16(u) || !aligned16(out) ||
        !aligned16(workspace) || !aligned4(page_table) || !aligned4(seqlens) ||
        (neff_out && !aligned4(neff_out)))
        return POLAR_ERR_INVALID_ARG;
    if (ws_bytes < decode_partials_bytes(num_seqs, max_pages, p->Hq, p->Hkv, 1))
        return POLAR_ERR_WORKSPACE;
    int *status = status_ptr();
    if (!status) return POLAR_ERR_CUDA;
    DecodeLaunch a;
    a.chunk = 1;
    a.per_head = 1;
    a.q = q; a.kv_pages = kv_pages; a.num_pages = num_pages; a.page_table = page_table;
    a.max_pages = max_pages; a.seqlens = seqlens; a.num_seqs = num_seqs; a.u = u; a.out = out;
    a.neff = neff_out; a.Hq = p->Hq; a.Hkv = p->Hkv; a.s = p->logit_scale; a.alpha = p->alpha;
    a.beta = p->beta; a.L = p->L_train; a.window = p->window; a.workspace = workspace;
    a.status = status;
    a.stream = static_cast<cudaStream_t>(stream);
    return from_cuda(launch_decode(a));
}

size_t polar_gdelta_prefill_workspace_size(const polar_gdelta_params_t *p) {
    if (check_gdelta_prefill(p) != POLAR_OK) return 0;
    return gdelta_workspace_bytes(p->B, p->T, p->H);
}

polar_status_t polar_gdelta_prefill(const void *q, const void *k, const void *v,
                                    const float *alpha, const float *beta, float *state,
                                    const polar_gdelta_params_t *p, void *out, void *workspace,
                                    size_t ws_bytes, void *stream) {
    polar_status_t st = check_gdelta_prefill(p);
    if (st != POLAR_OK) return st;
    if (p->B == 0 || p->T == 0) return POLAR_OK;
    if (!q || !k || !v || !alpha || !beta || !state || !out || !workspace)
        return POLAR_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(state) || !aligned16(out) ||
        !aligned16(workspace) || !aligned4(alpha) || !aligned4(beta))
        return POLAR_ERR_INVALID_ARG;
    if (ws_bytes < gdelta_workspace_bytes(p->B, p->T, p->H)) return POLAR_ERR_WORKSPACE;
    GdeltaLaunch a;
    a.q = q; a.k = k; a.v = v; a.alpha = alpha; a.beta = beta; a.state = state; a.out = out;
    a.B = p->B; a.T = p->T; a.H = p->H; a.dtype = p->dtype; a.zero_init = p->zero_init;
    a.accumulate = p->accumulate; a.workspace = workspace;
    a.stream = static_cast<cudaStream_t>(stream);
    return from_cuda(launch_gdelta_prefill(a));
}

polar_status_t polar_gdelta_step(const void *q, const void *k, const void *v,
                                 const float *alpha, const float *beta, float *state_pool,
                                 int num_slots, const int32_t *slots, int num_seqs,
                                 const polar_gdelta_params_t *p, void *out, void *stream) {
    polar_status_t st = check_gdelta(p);
    if (st != POLAR_OK) return st;
    if (num_seqs < 0 || num_slots < 0) return POLAR_ERR_INVALID_ARG;
    if (static_cast<long long>(num_seqs) * p->H > (1ll << 31) - 1) return POLAR_ERR_UNSUPPORTED;
    if (num_seqs == 0) return POLAR_OK;
    if (!q || !k || !v || !alpha || !beta || !slots || !out || (num_slots > 0 && !state_pool))
        return POLAR_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
        (state_pool && !aligned16(state_pool)) || !aligned4(alpha) || !aligned4(beta) ||
        !aligned4(slots))
        return POLAR_ERR_INVALID_ARG;
    int *status = status_ptr();
    if (!status) return POLAR_ERR_CUDA;
    GdeltaStepLaunch a;
    a.q = q; a.k = k; a.v = v; a.alpha = alpha; a.beta = beta; a.pool = state_pool;
    a.num_slots = num_slots; a.slots = slots; a.num_seqs = num_seqs; a.H = p->H;
    a.dtype = p->dtype; a.accumulate = p->accumulate; a.out = out; a.status = status;
    a.stream = static_cast<cudaStream_t>(stream);
    return from_cuda(launch_gdelta_step(a));
}

}  // extern "C"
