// gemv.cu -- CUDA-core expert-routed GEMV (decode path).
//
// For each expert that at least one (token, slot) pair selects, a CTA streams a
// block of that expert's packed weight rows once, dequantises the codes in
// registers, and accumulates the dot products with the x rows of every pair
// routed to the expert (up to NPB pairs per pass), x being staged once per CTA
// in shared memory. Each weight row is read with 16-byte loads by 8 lanes and
// reduced with warp shuffles. This is the decode design the pages argue for:
// x read once per block instead of once per output row (turboquant
// fast_switch_patch.py, module doc on polar_multi_gather_qmv) and weights read
// once for all rows of a batch (spark_model quant_dispatch.rs,
// w4a16_gemv_batch2/3/batchm), here without a cap on the number of pairs: an
// expert with more than NPB pairs is processed in several passes.
//
// Two routing modes:
//   fused  (R = m*n_expert_used <= 64): every CTA reads all ids, finds the
//          distinct experts in ascending order and the pairs of its own expert;
//          grid.y indexes the distinct experts.
//   routed (any R): grid.y indexes experts; counts / offsets / sorted_pairs come
//          from the routing prologue.
#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr int GEMV_THREADS = 256;
constexpr int GEMV_LPR = 8;                                      // lanes per row
constexpr int GEMV_ROWS = GEMV_THREADS / GEMV_LPR;               // 32 rows per CTA
constexpr uint32_t FUSED_MAX_R = 64;
constexpr int UNITS_PER_BATCH = 4;
constexpr size_t GEMV_SMEM_BUDGET = 200 * 1024;

// Words (u32) and codes per unit of each storage kind. A unit is the span a lane
// handles in one step: 16 bytes, or 48 bytes (64 codes) for 6-bit triplets.
template <int KIND> struct UnitShape;
template <> struct UnitShape<K_AFF4> { static constexpr int UW = 4, UC = 32; };
template <> struct UnitShape<K_AFF8> { static constexpr int UW = 4, UC = 16; };
template <> struct UnitShape<K_AFF6> { static constexpr int UW = 12, UC = 64; };
template <> struct UnitShape<K_CB2> { static constexpr int UW = 4, UC = 64; };
template <> struct UnitShape<K_CB3> { static constexpr int UW = 4, UC = 40; };
template <> struct UnitShape<K_CB4> { static constexpr int UW = 4, UC = 32; };
template <> struct UnitShape<K_NVFP4> { static constexpr int UW = 4, UC = 32; };

// Code i (compile-time) of a unit held in registers.
template <int KIND, int I, int UW>
__device__ __forceinline__ uint32_t unit_code(const uint32_t (&w)[UW]) {
    if constexpr (KIND == K_AFF4 || KIND == K_CB4 || KIND == K_NVFP4) {
        return (w[I / 8] >> (4 * (I % 8))) & 15u;
    } else if constexpr (KIND == K_AFF8) {
        return (w[I / 4] >> (8 * (I % 4))) & 255u;
    } else if constexpr (KIND == K_CB2) {
        return (w[I / 16] >> (2 * (I % 16))) & 3u;
    } else if constexpr (KIND == K_CB3) {
        return (w[I / 10] >> (3 * (I % 10))) & 7u;
    } else {  // K_AFF6: bit 6*I of the unit's little-endian bit string
        constexpr int b = 6 * I, wi = b / 32, sh = b % 32;
        if constexpr (sh <= 26) {
            return (w[wi] >> sh) & 63u;
        } else {
            return __funnelshift_r(w[wi], w[wi + 1], sh) & 63u;
        }
    }
}

// Load one unit's words. mode 16: 16-byte vector loads (row start 16-byte
// aligned and row_bytes % 16 == 0); mode 4: word loads (row_bytes % 4 == 0);
// mode 1: byte loads. Bytes at or beyond row_bytes read as zero.
template <int UW>
__device__ __forceinline__ void load_unit(const uint8_t *row, uint32_t unit, uint32_t row_bytes,
                                          int mode, uint32_t (&w)[UW]) {
    const uint32_t off = unit * (uint32_t)(UW * 4);
    if (mode == 16) {
#pragma unroll
        for (int v = 0; v < UW / 4; v++) {
            uint4 q = make_uint4(0, 0, 0, 0);
            if (off + 16u * v < row_bytes) q = __ldg((const uint4 *)(row + off) + v);
            w[4 * v] = q.x; w[4 * v + 1] = q.y; w[4 * v + 2] = q.z; w[4 * v + 3] = q.w;
        }
    } else if (mode == 4) {
#pragma unroll
        for (int v = 0; v < UW; v++)
            w[v] = (off + 4u * v < row_bytes) ? __ldg((const uint32_t *)(row + off) + v) : 0u;
    } else {
#pragma unroll
        for (int v = 0; v < UW; v++) {
            uint32_t x = 0;
#pragma unroll
            for (int b = 0; b < 4; b++) {
                uint32_t o = off + 4u * v + b;
                if (o < row_bytes) x |= (uint32_t)__ldg(row + o) << (8 * b);
            }
            w[v] = x;
        }
    }
}

struct GemvCtx {
    const uint8_t *row;       // packed row of (expert, col)
    const void *scales;       // row's scales
    const void *biases;       // row's biases (affine)
    const uint16_t *codebook; // codebook (f16 bits)
    uint32_t row_bytes, gs, groups;
};

template <int KIND>
__device__ __forceinline__ void load_group(const GemvCtx &c, uint32_t g, float &s, float &b) {
    g = min(g, c.groups - 1u);
    if constexpr (KIND == K_AFF4 || KIND == K_AFF6 || KIND == K_AFF8) {
        s = bf16_bits_to_f32(__ldg((const unsigned short *)c.scales + g));
        b = bf16_bits_to_f32(__ldg((const unsigned short *)c.biases + g));
    } else if constexpr (KIND == K_NVFP4) {
        s = e4m3_to_f32(__ldg((const uint8_t *)c.scales + g));
        b = 0.f;
    } else {
        s = f16_bits_to_f32(__ldg((const unsigned short *)c.scales + g));
        b = 0.f;
    }
}

template <int KIND>
__device__ __forceinline__ float dequant(uint32_t code, float s, float b, const float *cb) {
    if constexpr (KIND == K_AFF4 || KIND == K_AFF6 || KIND == K_AFF8) {
        return fmaf((float)code, s, b);
    } else if constexpr (KIND == K_NVFP4) {
        return e2m1_to_f32(code) * s;
    } else {
        return cb[code] * s;
    }
}

// Dot products of one unit with NPB staged x rows.
template <int KIND, int NPB, int I, int UW, int UC>
struct UnitDot {
    static __device__ __forceinline__ void run(const uint32_t (&w)[UW], const GemvCtx &c,
                                               uint32_t j0, uint32_t &g, uint32_t &gend, float &s,
                                               float &b, const float *xs, uint32_t xstride,
                                               const float *cb, float (&acc)[NPB]) {
        if constexpr (I < UC) {
            const uint32_t j = j0 + I;
            if (j >= gend) {
                g++;
                gend += c.gs;
                load_group<KIND>(c, g, s, b);
            }
            const float wv = dequant<KIND>(unit_code<KIND, I>(w), s, b, cb);
#pragma unroll
            for (int q = 0; q < NPB; q++) acc[q] = fmaf(wv, xs[q * xstride + I], acc[q]);
            UnitDot<KIND, NPB, I + 1, UW, UC>::run(w, c, j0, g, gend, s, b, xs, xstride, cb, acc);
        }
    }
};

struct GemvParams {
    const void *x;
    const uint32_t *ids;
    const uint8_t *packed;
    const void *scales;
    const void *aux;
    void *out;
    uint32_t *err;
    const uint32_t *counts, *offsets, *sorted_pairs;  // routed mode
    uint32_t R, k, n, gs, groups, n_expert_used, num_experts, row_bytes, n_units, xstride;
    int x_dtype, out_dtype, load_mode;
};

template <int KIND, int NPB, bool FUSED>
__global__ void __launch_bounds__(GEMV_THREADS)
gemv_kernel(const GemvParams P) {
    using U = UnitShape<KIND>;
    extern __shared__ float xs[];  // [NPB][xstride]
    __shared__ uint32_t ids_s[FUSED_MAX_R];
    __shared__ uint32_t first_s[FUSED_MAX_R];
    __shared__ uint32_t pairs_s[NPB];
    __shared__ uint32_t expert_s, npairs_s, pair_base_s;
    __shared__ float cb_s[16];

    const uint32_t tid = threadIdx.x;
    const uint32_t row0 = blockIdx.x * GEMV_ROWS;

    uint32_t expert = 0, total_pairs = 0;
    const uint32_t *pair_src = nullptr;  // routed mode: sorted pairs of this expert
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
            if (rank == blockIdx.y) expert_s = e;
        }
        if (tid == 0) {
            uint32_t D = 0;
            for (uint32_t t = 0; t < R; t++) D += first_s[t];
            npairs_s = D;  // temporarily: number of distinct experts
        }
        __syncthreads();
        // Zero the rows of out-of-range pairs (this row block) and flag them.
        if (blockIdx.y == 0) {
            for (uint32_t idx = tid; idx < R * GEMV_ROWS; idx += blockDim.x) {
                const uint32_t p = idx / GEMV_ROWS, r = row0 + idx % GEMV_ROWS;
                if (ids_s[p] >= E && r < P.n) store_out(P.out, P.out_dtype, (size_t)p * P.n + r, 0.f);
            }
            if (blockIdx.x == 0 && tid < R && ids_s[tid] >= E) atomicOr(P.err, ERR_BAD_ID);
        }
        if (blockIdx.y >= npairs_s) return;  // uniform
        expert = expert_s;
        __syncthreads();
        if (tid == 0) {
            uint32_t c = 0;
            for (uint32_t t = 0; t < R; t++) c += ids_s[t] == expert;
            npairs_s = c;
        }
        __syncthreads();
        total_pairs = npairs_s;
    } else {
        expert = blockIdx.y;
        total_pairs = __ldg(P.counts + expert);
        if (total_pairs == 0) return;
        pair_src = P.sorted_pairs + __ldg(P.offsets + expert);
    }

    if constexpr (KIND == K_CB2 || KIND == K_CB3 || KIND == K_CB4) {
        if (tid < (1u << kind_bits(KIND)))
            cb_s[tid] = f16_bits_to_f32(__ldg((const unsigned short *)P.aux + tid));
    }

    const uint32_t warp = tid >> 5, lane = tid & 31u;
    const uint32_t rsub = lane / GEMV_LPR, l8 = lane % GEMV_LPR;
    const uint32_t row = row0 + warp * (32 / GEMV_LPR) + rsub;
    const bool row_ok = row < P.n;
    const uint32_t row_c = row_ok ? row : P.n - 1;  // clamp: loads stay in bounds
    const size_t row_index = (size_t)expert * P.n + row_c;

    GemvCtx c;
    c.row = P.packed + row_index * P.row_bytes;
    c.row_bytes = P.row_bytes;
    c.gs = P.gs;
    c.groups = P.groups;
    c.codebook = (const uint16_t *)P.aux;
    if constexpr (KIND == K_NVFP4) {
        c.scales = (const uint8_t *)P.scales + row_index * P.groups;
        c.biases = nullptr;
    } else {
        c.scales = (const uint16_t *)P.scales + row_index * P.groups;
        c.biases = (KIND == K_AFF4 || KIND == K_AFF6 || KIND == K_AFF8)
                       ? (const void *)((const uint16_t *)P.aux + row_index * P.groups)
                       : nullptr;
    }
    const float s2 = (KIND == K_NVFP4) ? __ldg((const float *)P.aux + expert) : 1.f;

    for (uint32_t pb = 0; pb < total_pairs; pb += NPB) {
        const uint32_t np = tmin<uint32_t>(NPB, total_pairs - pb);
        __syncthreads();  // previous batch's x reads are done
        if (tid == 0) {
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
        __syncthreads();
        // Stage x rows: element j of pair q at xs[q*xstride + j + j/UC] (one pad word per unit).
        const uint32_t span = P.n_units * U::UC;
        for (uint32_t idx = tid; idx < NPB * span; idx += blockDim.x) {
            const uint32_t q = idx / span, j = idx % span;
            float v = 0.f;
            if (q < np && j < P.k) {
                const uint32_t t = pairs_s[q] / P.n_expert_used;
                v = load_x(P.x, P.x_dtype, (size_t)t * P.k + j);
            }
            xs[q * P.xstride + j + j / U::UC] = v;
        }
        __syncthreads();

        float acc[NPB];
#pragma unroll
        for (int q = 0; q < NPB; q++) acc[q] = 0.f;
        for (uint32_t u0 = l8; u0 < P.n_units; u0 += GEMV_LPR * UNITS_PER_BATCH) {
            uint32_t w[UNITS_PER_BATCH][U::UW];
#pragma unroll
            for (int ub = 0; ub < UNITS_PER_BATCH; ub++) {
                const uint32_t u = u0 + ub * GEMV_LPR;
                if (u < P.n_units) {
                    load_unit<U::UW>(c.row, u, c.row_bytes, P.load_mode, w[ub]);
                } else {
#pragma unroll
                    for (int v = 0; v < U::UW; v++) w[ub][v] = 0u;
                }
            }
#pragma unroll
            for (int ub = 0; ub < UNITS_PER_BATCH; ub++) {
                const uint32_t u = u0 + ub * GEMV_LPR;
                if (u < P.n_units) {
                    const uint32_t j0 = u * U::UC;
                    uint32_t g = j0 / c.gs, gend = (g + 1) * c.gs;
                    float s, b;
                    load_group<KIND>(c, g, s, b);
                    UnitDot<KIND, NPB, 0, U::UW, U::UC>::run(w[ub], c, j0, g, gend, s, b,
                                                             xs + u * (U::UC + 1), P.xstride,
                                                             cb_s, acc);
                }
            }
        }
#pragma unroll
        for (int q = 0; q < NPB; q++) {
#pragma unroll
            for (int d = GEMV_LPR / 2; d > 0; d >>= 1) acc[q] += __shfl_xor_sync(0xFFFFFFFFu, acc[q], d);
        }
        if (l8 == 0 && row_ok) {
#pragma unroll
            for (int q = 0; q < NPB; q++)
                if ((uint32_t)q < np)
                    store_out(P.out, P.out_dtype, (size_t)pairs_s[q] * P.n + row, acc[q] * s2);
        }
    }
}

template <int KIND, int NPB, bool FUSED>
cudaError_t launch_one(const GemvParams &P, dim3 grid, cudaStream_t st) {
    const size_t smem = (size_t)NPB * P.xstride * sizeof(float);
    auto kern = gemv_kernel<KIND, NPB, FUSED>;
    if (smem > 48 * 1024) {
        static int smem_set[64];
        cudaError_t e = ensure_dyn_smem(kern, smem, smem_set);
        if (e != cudaSuccess) return e;
    }
    kern<<<grid, GEMV_THREADS, smem, st>>>(P);
    return cudaGetLastError();
}

template <int KIND, bool FUSED>
cudaError_t launch_npb(const GemvParams &P, uint32_t npb, dim3 grid, cudaStream_t st) {
    // keep the staged x rows within the shared-memory budget
    const size_t row_bytes = (size_t)P.xstride * sizeof(float);
    while (npb > 1 && npb * row_bytes > GEMV_SMEM_BUDGET) npb >>= 1;
    if (row_bytes > GEMV_SMEM_BUDGET) return cudaErrorInvalidConfiguration;
    if (npb <= 1) return launch_one<KIND, 1, FUSED>(P, grid, st);
    if (npb <= 2) return launch_one<KIND, 2, FUSED>(P, grid, st);
    if (npb <= 4) return launch_one<KIND, 4, FUSED>(P, grid, st);
    return launch_one<KIND, 8, FUSED>(P, grid, st);
}

template <bool FUSED>
cudaError_t launch_kind(const GemvParams &P, int kind, uint32_t npb, dim3 grid, cudaStream_t st) {
    switch (kind) {
        case K_AFF4: return launch_npb<K_AFF4, FUSED>(P, npb, grid, st);
        case K_AFF6: return launch_npb<K_AFF6, FUSED>(P, npb, grid, st);
        case K_AFF8: return launch_npb<K_AFF8, FUSED>(P, npb, grid, st);
        case K_CB2: return launch_npb<K_CB2, FUSED>(P, npb, grid, st);
        case K_CB3: return launch_npb<K_CB3, FUSED>(P, npb, grid, st);
        case K_CB4: return launch_npb<K_CB4, FUSED>(P, npb, grid, st);
        case K_NVFP4: return launch_npb<K_NVFP4, FUSED>(P, npb, grid, st);
        default: return cudaErrorInvalidValue;
    }
}

int unit_codes(int kind) {
    switch (kind) {
        case K_AFF4: return UnitShape<K_AFF4>::UC;
        case K_AFF6: return UnitShape<K_AFF6>::UC;
        case K_AFF8: return UnitShape<K_AFF8>::UC;
        case K_CB2: return UnitShape<K_CB2>::UC;
        case K_CB3: return UnitShape<K_CB3>::UC;
        case K_CB4: return UnitShape<K_CB4>::UC;
        default: return UnitShape<K_NVFP4>::UC;
    }
}

int unit_bytes(int kind) { return kind == K_AFF6 ? 48 : 16; }

GemvParams make_params(const QmmArgs &a, uint32_t *err) {
    GemvParams P{};
    P.x = a.x; P.ids = a.ids; P.packed = a.packed; P.scales = a.scales; P.aux = a.aux;
    P.out = a.out; P.err = err;
    P.R = a.m * a.n_expert_used;
    P.k = a.k; P.n = a.n; P.gs = a.group_size; P.groups = a.groups;
    P.n_expert_used = a.n_expert_used; P.num_experts = a.num_experts; P.row_bytes = a.row_bytes;
    const uint32_t uc = (uint32_t)unit_codes(a.kind), ub = (uint32_t)unit_bytes(a.kind);
    // units covering the row's bytes (and so all k codes)
    P.n_units = (a.row_bytes + ub - 1) / ub;
    if ((uint64_t)P.n_units * uc < a.k) P.n_units = (a.k + uc - 1) / uc;
    P.xstride = P.n_units * (uc + 1);
    P.x_dtype = a.x_dtype; P.out_dtype = a.out_dtype;
    const bool al16 = ((uintptr_t)a.packed % 16 == 0) && (a.row_bytes % 16 == 0);
    const bool al4 = ((uintptr_t)a.packed % 4 == 0) && (a.row_bytes % 4 == 0);
    P.load_mode = al16 ? 16 : al4 ? 4 : 1;
    return P;
}

}  // namespace

cudaError_t launch_gemv_fused(const QmmArgs &a, uint32_t *err, cudaStream_t st) {
    GemvParams P = make_params(a, err);
    const uint32_t distinct_max = min(P.R, a.num_experts);
    dim3 grid((a.n + GEMV_ROWS - 1) / GEMV_ROWS, distinct_max);
    // pairs of one expert come from distinct tokens unless ids repeat inside a token
    const uint32_t npb = tmin<uint32_t>(a.m, 8u);
    return launch_kind<true>(P, a.kind, npb, grid, st);
}

cudaError_t launch_gemv_routed(const QmmArgs &a, const uint32_t *counts, const uint32_t *offsets,
                               const uint32_t *sorted_pairs, uint32_t *err, cudaStream_t st) {
    GemvParams P = make_params(a, err);
    P.counts = counts; P.offsets = offsets; P.sorted_pairs = sorted_pairs;
    dim3 grid((a.n + GEMV_ROWS - 1) / GEMV_ROWS, a.num_experts);
    return launch_kind<false>(P, a.kind, 8u, grid, st);
}

}  // namespace moe
