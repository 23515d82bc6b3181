// gemv_common.cuh -- pieces shared by the decode-path kernels: launch
// parameters and the routing prologue of one CTA (fused or routed).
#pragma once

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int GEMV_THREADS = 256;
constexpr int GEMV_LPR = 8;                         // lanes per row
constexpr int GEMV_ROWS = GEMV_THREADS / GEMV_LPR;  // 32 rows per CTA
constexpr uint32_t FUSED_MAX_R = 64;
constexpr size_t GEMV_SMEM_BUDGET = 200 * 1024;

struct GemvParams {
    const void *x;
    const uint32_t *ids;
    const uint8_t *packed;
    const void *scales;
    const void *aux;
    void *out;
    uint32_t *err;
    const uint32_t *counts, *offsets, *sorted_pairs;  // routed mode
    uint32_t R, m, k, n, gs, groups, n_expert_used, num_experts, row_bytes, n_units, xstride;
    int x_dtype, out_dtype, load_mode;
    int x_spec;        // TMA kernels: stage all m x rows before routing
    int s_bulk;        // one-token kernel: scale and bias rows staged by bulk copies
    const void *bias;  // per-expert output bias [num_experts, n] (bias_dtype), or null
    int bias_dtype;
    // pointer-table weights (null: contiguous [E, n, ...] arrays): per-expert base
    // addresses of the packed rows, scales and affine biases; a null packed pointer
    // means the expert is not held here and its pairs' rows are left untouched
    const uint64_t *packed_ptrs, *scale_ptrs, *bias_ptrs;
    // gated output (glu_nh = n/2; 0: plain): rows are walked in the logical order of
    // glu_row and out rows hold out_n = n/2 values act(gate) * up (else out_n = n)
    uint32_t glu_nh, out_n;
    int act;
    // programmatic dependent launch (one-token kernel): with early_weights the ids,
    // weights and scales are read, and the weight copies issued, before waiting for
    // the previous kernel on the stream; otherwise everything waits for it
    int pdl, early_weights;
    // failure-detection test hook (one-token kernel): non-zero makes every CTA first
    // wait this long on a barrier nothing completes, so that it aborts; 0 normally
    uint64_t fault_ns;
};

// Which expert this CTA serves and how many pairs it has. Fused mode: all ids
// are read into shared memory, distinct valid experts are ranked in ascending
// order and blockIdx.y picks one; CTAs with blockIdx.y == 0 also zero the rows
// of out-of-range pairs for their row block. Routed mode: blockIdx.y is the
// expert and its pairs come from the routing prologue. Returns false (for the
// whole CTA) when there is no work. Contains __syncthreads: call uniformly.
template <bool FUSED>
__device__ __forceinline__ bool route_prologue(const GemvParams &P, uint32_t *ids_s,
                                               uint32_t *first_s, uint32_t *expert_s,
                                               uint32_t *count_s, uint32_t row0, uint32_t rows,
                                               uint32_t &expert, uint32_t &total_pairs,
                                               const uint32_t *&pair_src) {
    const uint32_t tid = threadIdx.x;
    if constexpr (FUSED) {
        const uint32_t R = P.R, E = P.num_experts;
        if (tid < R) ids_s[tid] = __ldg(P.ids + tid);
        __syncthreads();
        if (tid < R) {
            const uint32_t e = ids_s[tid];
            bool first = e < E;
            for (uint32_t t = 0; t < tid && first; t++) first = ids_s[t] != e;
            first_s[tid] = first;
        }
        __syncthreads();
        if (tid < R && first_s[tid]) {
            const uint32_t e = ids_s[tid];
            uint32_t rank = 0;
            for (uint32_t t = 0; t < R; t++) rank += (first_s[t] && ids_s[t] < e);
            if (rank == blockIdx.y) *expert_s = e;
        }
        if (tid == 0) {
            uint32_t D = 0;
            for (uint32_t t = 0; t < R; t++) D += first_s[t];
            *count_s = D;  // number of distinct valid experts
        }
        __syncthreads();
        if (blockIdx.y == 0) {
            // output columns of this row block: half as many with a gated output
            const uint32_t sh = P.glu_nh ? 1u : 0u, c0 = row0 >> sh, cn = rows >> sh;
            for (uint32_t idx = tid; idx < R * cn; idx += blockDim.x) {
                const uint32_t p = idx / cn, c = c0 + idx % cn;
                if (ids_s[p] >= E && c < P.out_n) store_out(P.out, P.out_dtype, (size_t)p * P.out_n + c, 0.f);
            }
            if (blockIdx.x == 0 && tid < R && ids_s[tid] >= E) atomicOr(P.err, ERR_BAD_ID);
        }
        if (blockIdx.y >= *count_s) return false;  // uniform
        expert = *expert_s;
        __syncthreads();
        if (tid == 0) {
            uint32_t c = 0;
            for (uint32_t t = 0; t < R; t++) c += ids_s[t] == expert;
            *count_s = c;
        }
        __syncthreads();
        total_pairs = *count_s;
        return true;
    } else {
        expert = blockIdx.y;
        total_pairs = __ldg(P.counts + expert);
        if (total_pairs == 0) return false;
        pair_src = P.sorted_pairs + __ldg(P.offsets + expert);
        return true;
    }
}

// Pairs [pb, pb+np) of this CTA's expert into pairs_s (thread 0).
template <bool FUSED>
__device__ __forceinline__ void load_pairs(const GemvParams &P, const uint32_t *ids_s,
                                           uint32_t expert, const uint32_t *pair_src, uint32_t pb,
                                           uint32_t np, uint32_t *pairs_s) {
    if (threadIdx.x == 0) {
        if constexpr (FUSED) {
            uint32_t c2 = 0, seen = 0;
            for (uint32_t t = 0; t < P.R && c2 < np; t++)
                if (ids_s[t] == expert) {
                    if (seen >= pb) pairs_s[c2++] = t;
                    seen++;
                }
        } else {
            for (uint32_t q = 0; q < np; q++) pairs_s[q] = __ldg(pair_src + pb + q);
        }
    }
}


}  // namespace
}  // namespace moe
