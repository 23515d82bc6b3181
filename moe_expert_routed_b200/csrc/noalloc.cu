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
// the device address comes from cudaGetSymbolAddress, once per device and context.
static __device__ __align__(256) uint8_t g_noalloc_scratch[MOE_NOALLOC_SCRATCH_BYTES];

std::mutex g_scratch_mutex;

// Cached device address of the scratch per device, with the id of the CUDA
// context it was looked up in: a new context on the device (after
// cudaDeviceReset, or a caller's own context made current) loads the module
// again and the array may move, so the address is looked up again then.
struct ScratchAddr {
    void *ptr;
    unsigned long long ctx_id;
};
ScratchAddr g_scratch[64];

// cuCtxGetCurrent / cuCtxGetId through the runtime's driver entry points (no
// link-time dependency on the driver library).
typedef int (*ctx_get_current_t)(void **ctx);
typedef int (*ctx_get_id_t)(void *ctx, unsigned long long *id);
ctx_get_current_t g_ctx_get_current;
ctx_get_id_t g_ctx_get_id;
bool g_entry_points_looked_up;

// Unique id of the current context, or 0 when there is none or it cannot be read.
unsigned long long current_context_id() {
    if (!g_entry_points_looked_up) {
        g_entry_points_looked_up = true;
        cudaDriverEntryPointQueryResult q1, q2;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", (void **)&g_ctx_get_current, cudaEnableDefault, &q1) !=
                cudaSuccess || q1 != cudaDriverEntryPointSuccess)
            g_ctx_get_current = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", (void **)&g_ctx_get_id, cudaEnableDefault, &q2) !=
                cudaSuccess || q2 != cudaDriverEntryPointSuccess)
            g_ctx_get_id = nullptr;
    }
    if (!g_ctx_get_current || !g_ctx_get_id) return 0;
    void *ctx = nullptr;
    unsigned long long id = 0;
    if (g_ctx_get_current(&ctx) != 0 || !ctx) return 0;
    if (g_ctx_get_id(ctx, &id) != 0) return 0;
    return id;
}

// Device address of the scratch on the current device and context: looked up on
// the first call per device (and again whenever the current context differs from
// the one the cached address came from), with that device current.
moe_status scratch_address(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MOE_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    const unsigned long long id = current_context_id();
    if (!g_scratch[dev].ptr || id == 0 || id != g_scratch[dev].ctx_id) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return MOE_ERR_CUDA;
        g_scratch[dev].ptr = ptr;
        g_scratch[dev].ctx_id = current_context_id();  // the lookup may have created the context
    }
    *out = g_scratch[dev].ptr;
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

extern "C" moe_status moe_qmm_id_noalloc_poll_error(moe_stream_t stream) {
    void *scratch = nullptr;
    const moe_status s = scratch_address(&scratch);
    if (s != MOE_OK) return s;
    // the error word is the scratch's first word, as in a caller's workspace
    return moe_qmm_id_poll_error(scratch, stream);
}
