// internal.h -- launchers shared between the library's translation units.
#pragma once

#include <cuda_runtime.h>

#include "moe_qmm.h"
#include <stddef.h>
#include <stdint.h>

namespace moe {

// Routing prologue sizes.
constexpr uint32_t ROUTE_CHUNK = 4096;      // ids per histogram / scatter CTA
constexpr uint32_t ROUTE_THREADS = 256;
constexpr uint32_t ROUTE_MAX_E = 1024;      // experts (the out-of-range bucket is extra)

// Workspace layout (byte offsets; every section 256-byte aligned).
struct WsLayout {
    size_t err;          // u32 error word at offset 0
    size_t tile_count;   // u32
    size_t work_counter; // u32: the grouped GEMM's dynamic work counter (zeroed by the routing prologue)
    size_t counts;       // (E+1) u32
    size_t offsets;      // (E+2) u32
    size_t sorted_pairs; // R u32
    size_t tiles;        // max_tiles * 2 u32
    size_t chunk_hist;   // C * (E+1) u32
    size_t chunk_base;   // C * (E+1) u32
    size_t total;
    uint32_t max_tiles;
    uint32_t chunks;
};

// Smallest tile height the grouped path uses (sizes the tile list).
constexpr uint32_t MIN_TILE_ROWS = 64;

bool ws_layout(uint64_t R, uint32_t E, WsLayout *L);

// Routing prologue: histogram -> scan -> stable scatter (+ zero rows of
// out-of-range pairs when `out` is non-null; zeroes *work_counter when non-null).
cudaError_t launch_route(const uint32_t *ids, uint32_t R, uint32_t E, uint32_t tile_rows,
                         uint32_t *counts, uint32_t *offsets, uint32_t *sorted_pairs,
                         uint32_t *tiles, uint32_t *tile_count, uint32_t max_tiles,
                         uint32_t *chunk_hist, uint32_t *chunk_base, uint32_t chunks,
                         uint32_t *err, void *out, uint32_t n, int out_dtype, cudaStream_t st,
                         uint32_t *work_counter = nullptr);

// cudaFuncSetAttribute(MaxDynamicSharedMemorySize) once per kernel and device:
// `cache` is a per-kernel array of the largest size already set, per device.
template <typename K>
inline cudaError_t ensure_dyn_smem(K kern, size_t bytes, int (&cache)[64]) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64 && cache[dev] >= (int)bytes) return cudaSuccess;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess && dev >= 0 && dev < 64) cache[dev] = (int)bytes;
    return e;
}

struct QmmArgs {
    const void *x;
    const uint32_t *ids;
    const uint8_t *packed;
    const void *scales;
    const void *aux;
    void *out;
    uint32_t m, k, n, group_size, bits, n_expert_used, num_experts;
    int fmt, kind, x_dtype, out_dtype;
    uint32_t row_bytes, groups;
    const void *bias;  // per-expert output bias [num_experts, n] (bias_dtype), or null
    int bias_dtype;
    const uint64_t *packed_ptrs, *scale_ptrs, *bias_ptrs;  // pointer-table weights, or null
    int act;         // gated output: -1 none, else the activation (moe_act) of act(gate) * up
    uint32_t out_n;  // columns of an output row: n, or n / 2 with a gated output
    uint32_t launch_flags;  // MOE_LAUNCH_* bits of the path argument
    // failure-detection test hook (moe_qmm_test_inject_wait_timeout): when non-zero,
    // kernels with bounded waits make one wait per CTA on a barrier nothing
    // completes, giving up after this many ns; 0 in normal operation
    uint64_t fault_wait_ns;
    int x_copies;  // 1: the grouped GEMM's loader warps copy x rows (test hook)
    // W4A4 on the grouped GEMM: the GEMM takes x as these bf16 values and multiplies
    // each output by tok_scale[token] (null: x as given, no factor)
    const float *tok_scale;
};

// CUDA-core GEMV with routing fused in (R <= 64).
cudaError_t launch_gemv_fused(const QmmArgs &a, uint32_t *err, cudaStream_t st);
// CUDA-core GEMV over the routing prologue's output (any R).
cudaError_t launch_gemv_routed(const QmmArgs &a, const uint32_t *counts, const uint32_t *offsets,
                               const uint32_t *sorted_pairs, uint32_t *err, cudaStream_t st);

// f32 x rows in expert order for the grouped GEMM, as bf16 high halves in rows
// [0, R) and the bf16 roundings of the remainders in rows [R, 2R); k % 8 == 0.
cudaError_t launch_gather_x(const void *x, int x_dtype, const uint32_t *sorted_pairs, uint32_t R, uint32_t k,
                            uint32_t n_expert_used, uint16_t *xg, cudaStream_t st);
// W4A4 activations: per-token NVFP4 quantisation of x [m, k] (k % 16 == 0; any output
// may be null): codes [m, k/2] (8-byte aligned), E4M3 scales [m, k/16], per-token
// f32 scales [m], and x^ [m, k] f32.
// x16 (optional) [m, k]: e2m1(q) * e4m3(s) as bf16 (exact), x^ without the per-token factor.
cudaError_t launch_quant_act(const void *x, int x_dtype, uint32_t m, uint32_t k, uint8_t *codes, uint8_t *scales,
                             float *gscale, float *xhat, uint16_t *x16, cudaStream_t st);
// The grouped GEMM's B operand image for 16-bit x (tile-major, 128-byte-swizzled f16
// lines, [max_tiles][ceil(k/64)][tile_rows][128 B]) and, for bf16 x, the per-token
// powers of two tok_scale [m] the epilogue applies (img 16-byte aligned).
cudaError_t launch_x_image(const void *x, int x_dtype, uint32_t m, uint32_t k, const uint32_t *sorted_pairs,
                           const uint32_t *tiles, const uint32_t *tile_count, const uint32_t *offsets,
                           uint32_t n_expert_used, uint32_t tile_rows, uint32_t max_tiles, uint8_t *img,
                           float *tok_scale, cudaStream_t st);
uint64_t x_image_bytes(uint64_t R, uint32_t E, uint32_t k, uint32_t tile_rows);
// Bytes of the gathered x rows (0 when the grouped GEMM does not use them: 16-bit x
// is gathered by the GEMM's tensor copies straight from x).
uint64_t gathered_x_bytes(uint64_t R, uint32_t k, int x_dtype);

// W4A4 on the block-scaled MMA (NVFP4 weights, k % 256 == 0, contiguous, no bias or
// gated output): the activations' codes [m, k/2], E4M3 factors [m, k/16] and
// per-token scales [m] from launch_quant_act; tiles of up to 128 pairs.
bool w4a4_mma_supported(const QmmArgs &a);
cudaError_t launch_gemm_w4a4(const QmmArgs &a, const uint8_t *xcodes, const uint8_t *xscales, const float *gscale,
                             const uint32_t *offsets, const uint32_t *sorted_pairs, const uint32_t *tiles,
                             const uint32_t *tile_count, uint32_t max_tiles, uint32_t *err, uint32_t *work_counter,
                             cudaStream_t st);
// tcgen05 grouped GEMM over the routing prologue's tiles (xg: gathered f32 x rows, or null).
bool gemm_supported(const QmmArgs &a);
uint32_t gemm_tile_rows(const QmmArgs &a);
cudaError_t launch_gemm(const QmmArgs &a, const uint32_t *offsets, const uint32_t *sorted_pairs,
                        const uint32_t *tiles, const uint32_t *tile_count, uint32_t max_tiles,
                        uint32_t *err, uint32_t *work_counter, const uint16_t *xg, const uint8_t *ximg,
                        cudaStream_t st);

// moe_qmm_id's scalar validation (MOE_OK or the status moe_qmm_id would return).
moe_status validate_call(const void *x, const uint32_t *ids, const void *packed, const void *scales,
                         const void *aux, const void *out, uint32_t m, uint32_t k, uint32_t n,
                         uint32_t group_size, uint32_t bits, moe_fmt fmt, uint32_t n_expert_used,
                         uint32_t num_experts, moe_dtype x_dtype, moe_dtype out_dtype);

}  // namespace moe
