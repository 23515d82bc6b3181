// noalloc.cu -- moe_qmm_id_noalloc: the expert-routed quantized matmul for
// callers that cannot allocate device memory themselves.
//
// Some callers have no way to hand the library a workspace: an inference
// service that reserves all device memory once at start-up and forbids any
// allocation on the request path, a plug-in that runs inside another
// framework whose caching allocator owns the device memory (a raw cudaMalloc
// would bypass its accounting and can fail when its pool holds nearly all of
// the memory), or a thin C/FFI caller that only has the operation's own
// inputs and outputs. For them the routing prologue's scratch lives in a
// fixed-size array in device memory that is part of this library: every GPU
// that loads the library holds MOE_NOALLOC_SCRATCH_BYTES of it until the
// process exits, and no call allocates or frees anything.
#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "moe_qmm.h"

namespace {

// The shared scratch. Its name, used in host code, is only a host-side handle:
// the device address comes from cudaGetSymbolAddress, once per device.
static __device__ __align__(256) uint8_t g_noalloc_scratch[MOE_NOALLOC_SCRATCH_BYTES];

std::mutex g_scratch_mutex;
void *g_scratch_ptr[64];

// Device address of the scratch on the current device (looked up on the first
// call per device, with that device current).
moe_status scratch_address(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MOE_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (!g_scratch_ptr[dev]) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return MOE_ERR_CUDA;
        g_scratch_ptr[dev] = ptr;
    }
    *out = g_scratch_ptr[dev];
    return MOE_OK;
}

}  // namespace

extern "C" moe_status moe_qmm_id_noalloc(const void *x, const uint32_t *ids, const void *packed,
                                         const void *scales, const void *aux, void *out, uint32_t m,
                                         uint32_t k, uint32_t n, uint32_t group_size, uint32_t bits,
                                         moe_fmt fmt, uint32_t n_expert_used, uint32_t num_experts,
                                         moe_dtype x_dtype, moe_dtype out_dtype, moe_stream_t stream) {
    // argument errors first, before any CUDA call
    const moe_status v = moe::validate_call(x, ids, packed, scales, aux, out, m, k, n, group_size, bits,
                                            fmt, n_expert_used, num_experts, x_dtype, out_dtype);
    if (v != MOE_OK) return v;
    // the scratch must hold the routing prologue's buffers for these sizes
    const size_t need = moe_qmm_id_workspace_bytes(m, n_expert_used, num_experts);
    if (need == 0) return MOE_ERR_UNSUPPORTED;
    if (need > MOE_NOALLOC_SCRATCH_BYTES) return MOE_ERR_WORKSPACE_TOO_SMALL;
    void *scratch = nullptr;
    const moe_status s = scratch_address(&scratch);
    if (s != MOE_OK) return s;
    return moe_qmm_id_path(x, ids, packed, scales, aux, out, m, k, n, group_size, bits, fmt,
                           n_expert_used, num_experts, x_dtype, out_dtype, scratch,
                           MOE_NOALLOC_SCRATCH_BYTES, stream, MOE_PATH_AUTO);
}
