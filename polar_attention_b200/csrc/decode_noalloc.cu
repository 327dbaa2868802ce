// decode_noalloc.cu -- polar_attn_decode_paged_noalloc: the paged decode for
// callers that cannot allocate device memory.  The per-split scratch of the
// decode lives in a fixed file-scope device array instead of a caller-provided
// workspace; everything else is polar_attn_decode_paged itself.
#include <mutex>

#include "polar_common.cuh"
#include "polar_internal.h"

namespace {

// Split scratch of the no-alloc decode: one copy on every device that loads the
// library, held until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[POLAR_NOALLOC_SCRATCH_BYTES];

std::mutex g_scratch_mu;
constexpr int kMaxDevices = 64;
void *g_scratch_addr[kMaxDevices] = {nullptr};

// In host code g_noalloc_scratch names a host-side stand-in, not device memory,
// so the device address is looked up once per device, with that device current.
// The same first call also makes everything the later calls touch resident on
// the device: looking the address up loads this file's module (the array with
// it) under lazy module loading, and the status word and the decode kernels are
// loaded here too, so that later calls allocate no device memory at all.
polar_status_t scratch_on_current_device(void **addr) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return POLAR_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return POLAR_ERR_CUDA;
        if (!polar::device_status_word() || polar::decode_preload() != cudaSuccess)
            return POLAR_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *addr = g_scratch_addr[dev];
    return POLAR_OK;
}

}  // namespace

extern "C" polar_status_t polar_attn_decode_paged_noalloc(
    const void *q, const void *kv_pages, int num_pages, const int32_t *page_table, int max_pages,
    const int32_t *seqlens, int num_seqs, const float *u, const polar_params_t *params, void *out,
    float *neff_out, void *stream) {
    // polar_attn_decode_workspace_size is 0 for arguments it rejects; those are
    // reported by polar_attn_decode_paged below with the usual codes.
    if (polar_attn_decode_workspace_size(num_seqs, max_pages, params) > POLAR_NOALLOC_SCRATCH_BYTES)
        return POLAR_ERR_WORKSPACE;
    void *scratch = nullptr;
    const polar_status_t st = scratch_on_current_device(&scratch);
    if (st != POLAR_OK) return st;
    return polar_attn_decode_paged(q, kv_pages, num_pages, page_table, max_pages, seqlens,
                                   num_seqs, u, params, out, neff_out, scratch,
                                   POLAR_NOALLOC_SCRATCH_BYTES, stream);
}
