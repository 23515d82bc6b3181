// api.cu -- the C ABI (include/moe_qmm.h): argument validation, workspace
// layout, path choice and launches. Validation follows the rules of mlx-native
// quantized_matmul_id.rs (quantized_matmul_id: bits in the allowed set; m, k, n,
// group_size, n_expert_used, num_experts all > 0; InvalidArgument otherwise) and
// happens before any CUDA call.
#include <string.h>

#include <atomic>

#include "common.cuh"
#include "internal.h"
#include "moe_qmm.h"

namespace moe {

// Wait limit of the failure-detection test hook (0: off).
static std::atomic<uint64_t> g_fault_wait_ns{0};
static std::atomic<int> g_x_copies{0};

static inline size_t al256(size_t v) { return (v + 255) & ~(size_t)255; }

bool ws_layout(uint64_t R, uint32_t E, WsLayout *L) {
    if (R > 0xFFFFFFFFull || E >= 0xFFFFFFF0u) return false;
    size_t off = 0;
    L->err = 0;
    L->tile_count = 4;
    L->work_counter = 8;
    off = 256;
    L->counts = off; off += al256(4ull * (E + 1ull));
    L->offsets = off; off += al256(4ull * (E + 2ull));
    L->sorted_pairs = off; off += al256(4ull * R);
    const uint64_t max_tiles = R / MIN_TILE_ROWS + E + 1ull;
    if (max_tiles > 0xFFFFFFFFull) return false;
    L->max_tiles = (uint32_t)max_tiles;
    L->tiles = off; off += al256(8ull * max_tiles);
    const uint64_t chunks = (R + ROUTE_CHUNK - 1) / ROUTE_CHUNK;
    L->chunks = (uint32_t)chunks;
    L->chunk_hist = off; off += al256(4ull * chunks * (E + 1ull));
    L->chunk_base = off; off += al256(4ull * chunks * (E + 1ull));
    L->total = off;
    return true;
}

// W4A4 workspace ahead of the operation's own: x^ f32 [m, k], bf16 [m, k], f32 [m],
// codes [m, k/2], E4M3 factors [m, k/16].
size_t w4a4_front_bytes(uint32_t m, uint32_t k) {
    return al256((uint64_t)m * k * 4ull) + al256((uint64_t)m * k * 2ull) + al256((uint64_t)m * 4ull) +
           al256((uint64_t)m * k / 2ull) + al256((uint64_t)m * k / 16ull);
}

uint64_t gathered_x_bytes(uint64_t R, uint32_t k, int x_dtype) {
    if (k % 8u != 0 || x_dtype != DT_F32) return 0;
    return al256(R * k * 4ull);
}

static uint64_t row_bytes_of(int fmt, uint32_t bits, uint32_t k) {
    if (fmt == FMT_NVFP4 || fmt == FMT_MXFP4) return k / 2u;
    if (fmt == FMT_AFFINE && bits == 6) return ((uint64_t)k + 3) / 4 * 3;
    const uint32_t epw = 32u / bits;
    return ((uint64_t)k + epw - 1) / epw * 4;
}

}  // namespace moe

using namespace moe;

extern "C" {

size_t moe_packed_row_bytes(moe_fmt fmt, uint32_t bits, uint32_t k) {
    if (kind_of((int)fmt, (int)bits) < 0) return 0;
    if ((fmt == MOE_FMT_NVFP4 || fmt == MOE_FMT_MXFP4) && (k & 1u)) return 0;
    return (size_t)row_bytes_of((int)fmt, bits, k);
}

size_t moe_qmm_id_workspace_bytes(uint32_t m, uint32_t n_expert_used, uint32_t num_experts) {
    WsLayout L;
    if (!ws_layout((uint64_t)m * n_expert_used, num_experts, &L)) return 0;
    return L.total;
}

size_t moe_qmm_id_workspace_bytes_k(uint32_t m, uint32_t k, uint32_t n_expert_used, uint32_t num_experts,
                                    moe_dtype x_dtype) {
    WsLayout L;
    if ((int)x_dtype < 0 || (int)x_dtype > 2) return 0;
    const uint64_t R = (uint64_t)m * n_expert_used;
    if (!ws_layout(R, num_experts, &L)) return 0;
    if (x_dtype == MOE_F32) return L.total + (size_t)gathered_x_bytes(R, k, (int)x_dtype);
    // 16-bit x: room for the f16 image when the automatic path takes the grouped GEMM
    if (R <= MOE_DECODE_MAX_ROUTINGS || R <= (uint64_t)MOE_DECODE_MAX_PAIRS_PER_EXPERT * num_experts || k % 8u != 0)
        return L.total;
    if (R < 96ull * num_experts) return L.total;  // 64-pair tiles keep the row copies
    return L.total + (size_t)x_image_bytes(R, num_experts, k, 256u) + al256(4ull * m);
}

const char *moe_status_str(moe_status s) {
    switch (s) {
        case MOE_OK: return "ok";
        case MOE_ERR_INVALID_ARGUMENT: return "invalid argument";
        case MOE_ERR_UNSUPPORTED: return "valid arguments the library does not implement";
        case MOE_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
        case MOE_ERR_CUDA: return "CUDA error";
        case MOE_ERR_BAD_EXPERT_ID: return "an expert id was >= num_experts (its output rows are zero)";
        case MOE_ERR_TIMEOUT: return "a bounded device wait gave up; outputs are not valid";
        case MOE_ERR_BAD_EXPERT_POINTER:
            return "a pointer-table expert had a null or misaligned scale / bias buffer (its rows are untouched)";
    }
    return "unknown status";
}

static moe_status validate(const void *x, const uint32_t *ids, const void *packed,
                           const void *scales, const void *aux, const void *out, uint32_t m,
                           uint32_t k, uint32_t n, uint32_t group_size, uint32_t bits, moe_fmt fmt,
                           uint32_t n_expert_used, uint32_t num_experts, moe_dtype x_dtype,
                           moe_dtype out_dtype) {
    if (kind_of((int)fmt, (int)bits) < 0) return MOE_ERR_INVALID_ARGUMENT;
    if (!m || !k || !n || !group_size || !n_expert_used || !num_experts) return MOE_ERR_INVALID_ARGUMENT;
    if ((int)x_dtype < 0 || (int)x_dtype > 2 || (int)out_dtype < 0 || (int)out_dtype > 2)
        return MOE_ERR_INVALID_ARGUMENT;
    if (!x || !ids || !packed || !scales || !out) return MOE_ERR_INVALID_ARGUMENT;
    if (!aux && fmt != MOE_FMT_MXFP4) return MOE_ERR_INVALID_ARGUMENT;  // MXFP4 has no aux array
    if (fmt == MOE_FMT_NVFP4 && (group_size != 16 || (k & 1u))) return MOE_ERR_INVALID_ARGUMENT;
    if (fmt == MOE_FMT_MXFP4 && (group_size != 32 || (k & 1u))) return MOE_ERR_INVALID_ARGUMENT;
    if (k % group_size != 0) return MOE_ERR_UNSUPPORTED;
    if ((uint64_t)m * n_expert_used > 0x7FFFFFFFull) return MOE_ERR_UNSUPPORTED;
    if (row_bytes_of((int)fmt, bits, k) > 0xFFFFFFFFull) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

}  // extern "C"

namespace moe {
// The scalar checks moe_qmm_id runs first, for other entry points of the library.
moe_status validate_call(const void *x, const uint32_t *ids, const void *packed, const void *scales,
                         const void *aux, const void *out, uint32_t m, uint32_t k, uint32_t n,
                         uint32_t group_size, uint32_t bits, moe_fmt fmt, uint32_t n_expert_used,
                         uint32_t num_experts, moe_dtype x_dtype, moe_dtype out_dtype) {
    return validate(x, ids, packed, scales, aux, out, m, k, n, group_size, bits, fmt, n_expert_used,
                    num_experts, x_dtype, out_dtype);
}
}  // namespace moe

namespace moe {
namespace {

// Weights held as per-expert buffers (null: contiguous [E, n, ...] arrays).
struct PtrTables {
    const uint64_t *packed, *scales, *biases;
};

// W4A4: the activations to quantise and where each quantised form goes; run()
// writes only the forms the chosen path reads.
struct W4A4Front {
    const void *x;       // [m, k] of x_dtype
    int x_dtype;
    float *xhat;         // [m, k] f32 x^ (CUDA-core paths)
    uint16_t *x16;       // [m, k] bf16 e2m1(q) * e4m3(s) (grouped GEMM on the kind::f16 MMA)
    float *g;            // [m] per-token factors (grouped GEMM)
    uint8_t *codes;      // [m, k/2] E2M1 codes (block-scaled MMA)
    uint8_t *xs;         // [m, k/16] E4M3 block scales (block-scaled MMA)
};

// moe_qmm_id with an optional per-expert output bias (null: none), optional
// pointer-table weights and an optional gated output (act >= 0: act(gate) * up).
// With w4 (W4A4), x is w4->xhat, written here before the path's kernels.
moe_status run(const void *x, const uint32_t *ids, const void *packed, const void *scales, const void *aux,
               const void *bias, void *out, uint32_t m, uint32_t k, uint32_t n, uint32_t group_size,
               uint32_t bits, moe_fmt fmt, uint32_t n_expert_used, uint32_t num_experts, moe_dtype x_dtype,
               moe_dtype out_dtype, moe_dtype bias_dtype, void *workspace, size_t workspace_bytes,
               moe_stream_t stream, moe_path path, PtrTables pt = {nullptr, nullptr, nullptr}, int act = -1,
               const W4A4Front *w4 = nullptr) {
    moe_status v = validate(x, ids, pt.packed ? (const void *)pt.packed : packed,
                            pt.packed ? (const void *)pt.scales : scales, aux, out, m, k, n, group_size, bits,
                            fmt, n_expert_used, num_experts, x_dtype, out_dtype);
    if (v != MOE_OK) return v;
    // the low byte is the path, higher bits launch flags
    const uint32_t launch_flags = (uint32_t)path & ~0xFFu;
    path = (moe_path)((uint32_t)path & 0xFFu);
    if ((int)path > 2 || (launch_flags & ~(uint32_t)(MOE_LAUNCH_PDL | MOE_LAUNCH_EARLY_WEIGHTS)))
        return MOE_ERR_INVALID_ARGUMENT;
    if (!workspace || ((uintptr_t)workspace & 15u)) return MOE_ERR_INVALID_ARGUMENT;
    const uint64_t R = (uint64_t)m * n_expert_used;
    WsLayout L;
    if (!ws_layout(R, num_experts, &L)) return MOE_ERR_UNSUPPORTED;
    if (workspace_bytes < L.total) return MOE_ERR_WORKSPACE_TOO_SMALL;

    QmmArgs a;
    a.x = x; a.ids = ids; a.packed = (const uint8_t *)packed; a.scales = scales; a.aux = aux;
    a.out = out; a.m = m; a.k = k; a.n = n; a.group_size = group_size; a.bits = bits;
    a.n_expert_used = n_expert_used; a.num_experts = num_experts;
    a.fmt = (int)fmt; a.kind = kind_of((int)fmt, (int)bits);
    a.x_dtype = (int)x_dtype; a.out_dtype = (int)out_dtype;
    a.row_bytes = (uint32_t)row_bytes_of((int)fmt, bits, k);
    a.groups = (k + group_size - 1) / group_size;
    a.bias = bias;
    a.bias_dtype = (int)bias_dtype;
    a.packed_ptrs = pt.packed;
    a.scale_ptrs = pt.scales;
    a.bias_ptrs = pt.biases;
    a.act = act;
    a.out_n = act >= 0 ? n / 2u : n;
    a.launch_flags = launch_flags;
    a.fault_wait_ns = g_fault_wait_ns.load(std::memory_order_relaxed);
    a.x_copies = g_x_copies.load(std::memory_order_relaxed);
    a.tok_scale = nullptr;

    uint8_t *ws = (uint8_t *)workspace;
    uint32_t *err = (uint32_t *)(ws + L.err);
    cudaStream_t st = (cudaStream_t)stream;
    const bool routable = num_experts <= ROUTE_MAX_E;
    const bool small = R <= MOE_DECODE_MAX_ROUTINGS;
    // few pairs per expert: the CUDA-core GEMV reads each expert's rows once for all
    // of its pairs and is faster than the tensor-core GEMM (measured crossover)
    const bool sparse = R <= (uint64_t)MOE_DECODE_MAX_PAIRS_PER_EXPERT * num_experts;

    enum { FUSED, ROUTED_GEMV, GROUPED } choice;
    if (path == MOE_PATH_GROUPED) {
        if (!routable || !gemm_supported(a)) return MOE_ERR_UNSUPPORTED;
        choice = GROUPED;
    } else if (path == MOE_PATH_DECODE) {
        if (small) choice = FUSED;
        else if (routable) choice = ROUTED_GEMV;
        else return MOE_ERR_UNSUPPORTED;
    } else {
        if (small) choice = FUSED;
        else if (routable && sparse) choice = ROUTED_GEMV;
        else if (routable && gemm_supported(a)) choice = GROUPED;
        else if (routable) choice = ROUTED_GEMV;
        else return MOE_ERR_UNSUPPORTED;
    }

    // W4A4 on the grouped GEMM: the block-scaled MMA on the activations' NVFP4 codes
    // where it applies; else bf16 e2m1(q) * e4m3(s) (exact) as the B operand and the
    // per-token factor in the epilogue, instead of the f32 x^ the CUDA-core paths take
    const bool w4mma = w4 && choice == GROUPED && !a.x_copies && w4a4_mma_supported(a);
    const bool w4x16 = w4 && choice == GROUPED && !w4mma;
    if (w4x16) {
        a.x = w4->x16;
        a.x_dtype = DT_BF16;
        x = w4->x16;
        x_dtype = MOE_BF16;
        a.tok_scale = w4->g;
        if (!gemm_supported(a)) return MOE_ERR_UNSUPPORTED;
    }
    if (w4 && moe::launch_quant_act(w4->x, w4->x_dtype, m, k, w4mma ? w4->codes : nullptr,
                                    w4mma ? w4->xs : nullptr, (w4mma || w4x16) ? w4->g : nullptr,
                                    (w4mma || w4x16) ? nullptr : w4->xhat, w4x16 ? w4->x16 : nullptr,
                                    (cudaStream_t)stream) != cudaSuccess)
        return MOE_ERR_CUDA;

    cudaError_t ce;
    if (choice == FUSED) {
        ce = launch_gemv_fused(a, err, st);
    } else {
        uint32_t *counts = (uint32_t *)(ws + L.counts);
        uint32_t *offsets = (uint32_t *)(ws + L.offsets);
        uint32_t *sp = (uint32_t *)(ws + L.sorted_pairs);
        uint32_t *tiles = (uint32_t *)(ws + L.tiles);
        uint32_t *tc = (uint32_t *)(ws + L.tile_count);
        const uint32_t tile_rows = w4mma ? 128u : choice == GROUPED ? gemm_tile_rows(a) : MIN_TILE_ROWS;
        const uint32_t max_tiles = (uint32_t)(R / tile_rows + num_experts + 1);
        uint32_t *wc = (uint32_t *)(ws + L.work_counter);
        // x rows in expert order for the grouped GEMM, when the workspace has room for them
        const uint64_t gx = (choice == GROUPED && !w4mma) ? gathered_x_bytes(R, k, (int)x_dtype) : 0;
        uint16_t *xg = (gx && workspace_bytes >= L.total + gx) ? (uint16_t *)(ws + L.total) : nullptr;
        // 16-bit x with 256-pair tiles: the tile-major f16 image of the B operand (and
        // bf16's per-token powers of two), when the workspace has room; not for MXFP4
        // (e2m1 * 2^e can leave f16's range), pointer tables, gated outputs or W4A4's
        // operand. With 64-pair tiles (a few pairs per expert) writing the image costs
        // more than the GEMM saves.
        uint8_t *ximg = nullptr;
        float *tscale = nullptr;
        if (choice == GROUPED && !w4mma && tile_rows == 256u && x_dtype != MOE_F32 && a.kind != K_MXFP4 &&
            !a.packed_ptrs && a.act < 0 && !a.tok_scale && !a.x_copies && ((uintptr_t)x & 15u) == 0) {
            const uint64_t ib = x_image_bytes(R, num_experts, k, tile_rows);
            if (workspace_bytes >= L.total + ib + al256(4ull * m)) {
                ximg = ws + L.total;
                tscale = (float *)(ws + L.total + ib);
            }
        }
        ce = launch_route(ids, (uint32_t)R, num_experts, tile_rows, counts, offsets, sp, tiles, tc,
                          max_tiles, (uint32_t *)(ws + L.chunk_hist),
                          (uint32_t *)(ws + L.chunk_base), L.chunks, err, out, a.out_n, (int)out_dtype,
                          st, wc);
        if (ce == cudaSuccess && xg) ce = launch_gather_x(x, (int)x_dtype, sp, (uint32_t)R, k, n_expert_used, xg, st);
        if (ce == cudaSuccess && ximg) {
            ce = launch_x_image(x, (int)x_dtype, m, k, sp, tiles, tc, offsets, n_expert_used, tile_rows, max_tiles,
                                ximg, tscale, st);
            a.x_dtype = DT_F16;
            a.tok_scale = x_dtype == MOE_BF16 ? tscale : nullptr;
        }
        if (ce == cudaSuccess) {
            if (w4mma)
                ce = launch_gemm_w4a4(a, w4->codes, w4->xs, w4->g, offsets, sp, tiles, tc, max_tiles,
                                      err, wc, st);
            else if (choice == GROUPED)
                ce = launch_gemm(a, offsets, sp, tiles, tc, max_tiles, err, wc, xg, ximg, st);
            else
                ce = launch_gemv_routed(a, counts, offsets, sp, err, st);
        }
    }
    return ce == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace
}  // namespace moe

extern "C" {

moe_status moe_qmm_id_path(const void *x, const uint32_t *ids, const void *packed,
                           const void *scales, const void *aux, void *out, uint32_t m, uint32_t k,
                           uint32_t n, uint32_t group_size, uint32_t bits, moe_fmt fmt,
                           uint32_t n_expert_used, uint32_t num_experts, moe_dtype x_dtype,
                           moe_dtype out_dtype, void *workspace, size_t workspace_bytes,
                           moe_stream_t stream, moe_path path) {
    return run(x, ids, packed, scales, aux, nullptr, out, m, k, n, group_size, bits, fmt, n_expert_used,
               num_experts, x_dtype, out_dtype, MOE_F32, workspace, workspace_bytes, stream, path);
}

moe_status moe_qmm_id_bias(const void *x, const uint32_t *ids, const void *packed, const void *scales,
                           const void *aux, const void *expert_bias, void *out, uint32_t m, uint32_t k,
                           uint32_t n, uint32_t group_size, uint32_t bits, moe_fmt fmt,
                           uint32_t n_expert_used, uint32_t num_experts, moe_dtype x_dtype,
                           moe_dtype out_dtype, moe_dtype bias_dtype, void *workspace,
                           size_t workspace_bytes, moe_stream_t stream, moe_path path) {
    if (!expert_bias || (int)bias_dtype < 0 || (int)bias_dtype > 2) return MOE_ERR_INVALID_ARGUMENT;
    return run(x, ids, packed, scales, aux, expert_bias, out, m, k, n, group_size, bits, fmt, n_expert_used,
               num_experts, x_dtype, out_dtype, bias_dtype, workspace, workspace_bytes, stream, path);
}

moe_status moe_qmm_id_ptrs(const void *x, const uint32_t *ids, const uint64_t *packed_ptrs,
                           const uint64_t *scale_ptrs, const uint64_t *bias_ptrs, const void *aux, void *out,
                           uint32_t m, uint32_t k, uint32_t n, uint32_t group_size, uint32_t bits, moe_fmt fmt,
                           uint32_t n_expert_used, uint32_t num_experts, moe_dtype x_dtype, moe_dtype out_dtype,
                           void *workspace, size_t workspace_bytes, moe_stream_t stream, moe_path path) {
    if (!packed_ptrs || !scale_ptrs || (fmt == MOE_FMT_AFFINE && !bias_ptrs)) return MOE_ERR_INVALID_ARGUMENT;
    // affine biases come from bias_ptrs; aux is the codebook or scale2 table
    const void *aux_arg = fmt == MOE_FMT_AFFINE ? (const void *)bias_ptrs : aux;
    return run(x, ids, nullptr, nullptr, aux_arg, nullptr, out, m, k, n, group_size, bits, fmt, n_expert_used,
               num_experts, x_dtype, out_dtype, MOE_F32, workspace, workspace_bytes, stream, path,
               PtrTables{packed_ptrs, scale_ptrs, bias_ptrs});
}

moe_status moe_qmm_id_glu(const void *x, const uint32_t *ids, const void *packed, const void *scales,
                          const void *aux, const void *expert_bias, void *out, uint32_t m, uint32_t k,
                          uint32_t n, uint32_t group_size, uint32_t bits, moe_fmt fmt,
                          uint32_t n_expert_used, uint32_t num_experts, moe_dtype x_dtype,
                          moe_dtype out_dtype, moe_dtype bias_dtype, moe_act act, void *workspace,
                          size_t workspace_bytes, moe_stream_t stream, moe_path path) {
    if ((int)act < 0 || (int)act > 2 || (n & 1u)) return MOE_ERR_INVALID_ARGUMENT;
    if (expert_bias && ((int)bias_dtype < 0 || (int)bias_dtype > 2)) return MOE_ERR_INVALID_ARGUMENT;
    return run(x, ids, packed, scales, aux, expert_bias, out, m, k, n, group_size, bits, fmt, n_expert_used,
               num_experts, x_dtype, out_dtype, expert_bias ? bias_dtype : MOE_F32, workspace, workspace_bytes,
               stream, path, PtrTables{nullptr, nullptr, nullptr}, (int)act);
}

size_t moe_qmm_id_workspace_bytes_w4a4(uint32_t m, uint32_t k, uint32_t n_expert_used, uint32_t num_experts) {
    const size_t rest = moe_qmm_id_workspace_bytes(m, n_expert_used, num_experts);
    if (!rest) return 0;
    return moe::al256(rest) + moe::w4a4_front_bytes(m, k);
}

moe_status moe_quantize_act_nvfp4(const void *x, uint32_t m, uint32_t k, moe_dtype x_dtype, uint8_t *codes,
                                  uint8_t *scales, float *gscale, float *xhat, moe_stream_t stream) {
    if (!x || m == 0 || k == 0 || (int)x_dtype < 0 || (int)x_dtype > 2) return MOE_ERR_INVALID_ARGUMENT;
    if (((uintptr_t)codes & 3u) || ((uintptr_t)xhat & 15u) || ((uintptr_t)gscale & 3u))
        return MOE_ERR_INVALID_ARGUMENT;
    if (k % 16u != 0) return MOE_ERR_UNSUPPORTED;
    return moe::launch_quant_act(x, (int)x_dtype, m, k, codes, scales, gscale, xhat, nullptr,
                                 (cudaStream_t)stream) ==
                   cudaSuccess
               ? MOE_OK
               : MOE_ERR_CUDA;
}

moe_status moe_qmm_id_w4a4(const void *x, const uint32_t *ids, const void *packed, const void *scales,
                           const void *aux, void *out, uint32_t m, uint32_t k, uint32_t n, uint32_t group_size,
                           uint32_t bits, moe_fmt fmt, uint32_t n_expert_used, uint32_t num_experts,
                           moe_dtype x_dtype, moe_dtype out_dtype, void *workspace, size_t workspace_bytes,
                           moe_stream_t stream, moe_path path) {
    moe_status v = moe::validate_call(x, ids, packed, scales, aux, out, m, k, n, group_size, bits, fmt,
                                      n_expert_used, num_experts, x_dtype, out_dtype);
    if (v != MOE_OK) return v;
    if (k % 16u != 0) return MOE_ERR_UNSUPPORTED;
    if (!workspace || ((uintptr_t)workspace & 15u)) return MOE_ERR_INVALID_ARGUMENT;
    // the operation's own workspace first (its error word at the start, as for
    // moe_qmm_id), then, from the last 256-byte boundary that leaves room for them,
    // x^ (f32), the bf16 values without the per-token factor, the per-token factors,
    // the E2M1 codes and the E4M3 block scales
    const size_t front = moe::w4a4_front_bytes(m, k);
    if (workspace_bytes < front) return MOE_ERR_WORKSPACE_TOO_SMALL;
    const size_t own = (workspace_bytes - front) & ~(size_t)255;
    if (own < moe_qmm_id_workspace_bytes(m, n_expert_used, num_experts)) return MOE_ERR_WORKSPACE_TOO_SMALL;
    uint8_t *w = (uint8_t *)workspace + own;
    size_t o = 0;
    float *xhat = (float *)(w + o);
    o += moe::al256((uint64_t)m * k * 4ull);
    uint16_t *x16 = (uint16_t *)(w + o);
    o += moe::al256((uint64_t)m * k * 2ull);
    float *g = (float *)(w + o);
    o += moe::al256((uint64_t)m * 4ull);
    uint8_t *codes = w + o;
    o += moe::al256((uint64_t)m * k / 2ull);
    uint8_t *xs = w + o;
    const moe::W4A4Front w4{x, (int)x_dtype, xhat, x16, g, codes, xs};
    return moe::run(xhat, ids, packed, scales, aux, nullptr, out, m, k, n, group_size, bits, fmt, n_expert_used,
                    num_experts, MOE_F32, out_dtype, MOE_F32, workspace, own, stream, path,
                    {nullptr, nullptr, nullptr}, -1, &w4);
}

moe_status moe_qmm_id(const void *x, const uint32_t *ids, const void *packed, const void *scales,
                      const void *aux, void *out, uint32_t m, uint32_t k, uint32_t n,
                      uint32_t group_size, uint32_t bits, moe_fmt fmt, uint32_t n_expert_used,
                      uint32_t num_experts, moe_dtype x_dtype, moe_dtype out_dtype,
                      void *workspace, size_t workspace_bytes, moe_stream_t stream) {
    return moe_qmm_id_path(x, ids, packed, scales, aux, out, m, k, n, group_size, bits, fmt,
                           n_expert_used, num_experts, x_dtype, out_dtype, workspace,
                           workspace_bytes, stream, MOE_PATH_AUTO);
}

}  // extern "C"

namespace moe {
namespace {

// What a moe_qmm_plan holds (inside the caller's opaque storage).
struct PlanData {
    uint64_t magic;
    const void *packed, *scales, *aux, *bias;
    void *workspace;
    size_t workspace_bytes;
    uint32_t m, k, n, group_size, bits, n_expert_used, num_experts;
    int32_t fmt, x_dtype, out_dtype, bias_dtype, act;
    uint32_t path;
};
static_assert(sizeof(PlanData) <= sizeof(moe_qmm_plan), "plan storage too small");
constexpr uint64_t PLAN_MAGIC = 0x6d6f65706c616e31ull;

}  // namespace
}  // namespace moe

extern "C" {

moe_status moe_qmm_plan_init(moe_qmm_plan *plan, const void *packed, const void *scales, const void *aux,
                             const void *expert_bias, uint32_t m, uint32_t k, uint32_t n,
                             uint32_t group_size, uint32_t bits, moe_fmt fmt, uint32_t n_expert_used,
                             uint32_t num_experts, moe_dtype x_dtype, moe_dtype out_dtype,
                             moe_dtype bias_dtype, int32_t act, void *workspace, size_t workspace_bytes,
                             moe_path path) {
    if (!plan) return MOE_ERR_INVALID_ARGUMENT;
    memset(plan, 0, sizeof(*plan));
    // the operation's checks, with placeholders for the per-call pointers
    const void *ph = packed;
    moe_status v = validate(ph, (const uint32_t *)ph, packed, scales, aux, ph, m, k, n, group_size, bits, fmt,
                            n_expert_used, num_experts, x_dtype, out_dtype);
    if (v != MOE_OK) return v;
    if (act < -1 || act > 2 || (act >= 0 && (n & 1u))) return MOE_ERR_INVALID_ARGUMENT;
    if (expert_bias && ((int)bias_dtype < 0 || (int)bias_dtype > 2)) return MOE_ERR_INVALID_ARGUMENT;
    const uint32_t flags = (uint32_t)path & ~0xFFu;
    if (((uint32_t)path & 0xFFu) > 2 || (flags & ~(uint32_t)(MOE_LAUNCH_PDL | MOE_LAUNCH_EARLY_WEIGHTS)))
        return MOE_ERR_INVALID_ARGUMENT;
    if (!workspace || ((uintptr_t)workspace & 15u)) return MOE_ERR_INVALID_ARGUMENT;
    WsLayout L;
    if (!ws_layout((uint64_t)m * n_expert_used, num_experts, &L)) return MOE_ERR_UNSUPPORTED;
    if (workspace_bytes < L.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
    PlanData d = {};
    d.packed = packed; d.scales = scales; d.aux = aux; d.bias = expert_bias;
    d.workspace = workspace; d.workspace_bytes = workspace_bytes;
    d.m = m; d.k = k; d.n = n; d.group_size = group_size; d.bits = bits;
    d.n_expert_used = n_expert_used; d.num_experts = num_experts;
    d.fmt = (int32_t)fmt; d.x_dtype = (int32_t)x_dtype; d.out_dtype = (int32_t)out_dtype;
    d.bias_dtype = expert_bias ? (int32_t)bias_dtype : (int32_t)MOE_F32;
    d.act = act; d.path = (uint32_t)path;
    d.magic = PLAN_MAGIC;
    memcpy(plan, &d, sizeof(d));
    return MOE_OK;
}

moe_status moe_qmm_plan_run(const moe_qmm_plan *plan, const void *x, const uint32_t *ids, void *out,
                            moe_stream_t stream) {
    if (!plan) return MOE_ERR_INVALID_ARGUMENT;
    PlanData d;
    memcpy(&d, plan, sizeof(d));
    if (d.magic != PLAN_MAGIC) return MOE_ERR_INVALID_ARGUMENT;
    return run(x, ids, d.packed, d.scales, d.aux, d.bias, out, d.m, d.k, d.n, d.group_size, d.bits,
               (moe_fmt)d.fmt, d.n_expert_used, d.num_experts, (moe_dtype)d.x_dtype, (moe_dtype)d.out_dtype,
               (moe_dtype)d.bias_dtype, d.workspace, d.workspace_bytes, stream, (moe_path)d.path,
               PtrTables{nullptr, nullptr, nullptr}, d.act);
}

moe_status moe_qmm_id_route(const uint32_t *ids, uint32_t m, uint32_t n_expert_used,
                            uint32_t num_experts, uint32_t tile_rows, uint32_t *counts,
                            uint32_t *offsets, uint32_t *sorted_pairs, uint32_t *tiles,
                            uint32_t *tile_count, void *workspace, size_t workspace_bytes,
                            moe_stream_t stream) {
    if (!m || !n_expert_used || !num_experts || !tile_rows || tile_rows > 65536u)
        return MOE_ERR_INVALID_ARGUMENT;
    if (!ids || !counts || !offsets || !sorted_pairs || !tiles || !tile_count || !workspace)
        return MOE_ERR_INVALID_ARGUMENT;
    if ((uintptr_t)workspace & 15u) return MOE_ERR_INVALID_ARGUMENT;
    if (num_experts > ROUTE_MAX_E) return MOE_ERR_UNSUPPORTED;
    const uint64_t R = (uint64_t)m * n_expert_used;
    if (R > 0x7FFFFFFFull) return MOE_ERR_UNSUPPORTED;
    WsLayout L;
    if (!ws_layout(R, num_experts, &L)) return MOE_ERR_UNSUPPORTED;
    if (workspace_bytes < L.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
    uint8_t *ws = (uint8_t *)workspace;
    const uint32_t max_tiles = (uint32_t)(R / tile_rows + num_experts + 1);
    cudaError_t ce = launch_route(ids, (uint32_t)R, num_experts, tile_rows, counts, offsets,
                                  sorted_pairs, tiles, tile_count, max_tiles,
                                  (uint32_t *)(ws + L.chunk_hist), (uint32_t *)(ws + L.chunk_base),
                                  L.chunks, (uint32_t *)(ws + L.err), nullptr, 0, 0,
                                  (cudaStream_t)stream);
    return ce == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status moe_qmm_test_inject_wait_timeout(uint64_t limit_ns) {
    moe::g_fault_wait_ns.store(limit_ns, std::memory_order_relaxed);
    return MOE_OK;
}

moe_status moe_qmm_test_x_copies(int on) {
    if (on != 0 && on != 1) return MOE_ERR_INVALID_ARGUMENT;
    moe::g_x_copies.store(on, std::memory_order_relaxed);
    return MOE_OK;
}

moe_status moe_qmm_id_poll_error(void *workspace, moe_stream_t stream) {
    if (!workspace) return MOE_ERR_INVALID_ARGUMENT;
    cudaStream_t st = (cudaStream_t)stream;
    uint32_t w = 0;
    if (cudaMemcpyAsync(&w, workspace, sizeof(w), cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return MOE_ERR_CUDA;
    if (w) {
        if (cudaMemsetAsync(workspace, 0, sizeof(w), st) != cudaSuccess) return MOE_ERR_CUDA;
        if (cudaStreamSynchronize(st) != cudaSuccess) return MOE_ERR_CUDA;
    }
    if (w & ERR_TIMEOUT) return MOE_ERR_TIMEOUT;
    if (w & ERR_BAD_ID) return MOE_ERR_BAD_EXPERT_ID;
    if (w & ERR_BAD_POINTER) return MOE_ERR_BAD_EXPERT_POINTER;
    if (w & ERR_INTERNAL) return MOE_ERR_CUDA;
    return MOE_OK;
}

}  // extern "C"
