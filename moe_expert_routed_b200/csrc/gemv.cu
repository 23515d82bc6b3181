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
#include "gemv_common.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace moe {

namespace {

__device__ __forceinline__ uint32_t ptx_smem_addr(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

constexpr int UNITS_PER_BATCH = 4;

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
template <> struct UnitShape<K_MXFP4> { static constexpr int UW = 4, UC = 32; };

// Code i (compile-time) of a unit held in registers.
template <int KIND, int I, int UW>
__device__ __forceinline__ uint32_t unit_code(const uint32_t (&w)[UW]) {
    if constexpr (KIND == K_AFF4 || KIND == K_CB4 || KIND == K_NVFP4 || KIND == K_MXFP4) {
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
    } else if constexpr (KIND == K_MXFP4) {
        s = e8m0_to_f32(__ldg((const uint8_t *)c.scales + g));
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
    } else if constexpr (KIND == K_NVFP4 || KIND == K_MXFP4) {
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



template <int KIND, int NPB, bool FUSED>
__global__ void __launch_bounds__(GEMV_THREADS)
gemv_kernel(const GemvParams P) {
    using U = UnitShape<KIND>;
    extern __shared__ float xs[];  // [NPB][xstride]
    __shared__ uint32_t ids_s[FUSED_MAX_R];
    __shared__ uint32_t first_s[FUSED_MAX_R];
    __shared__ uint32_t pairs_s[NPB];
    __shared__ uint32_t expert_s, npairs_s;
    __shared__ float cb_s[16];

    const uint32_t tid = threadIdx.x;
    const uint32_t row0 = blockIdx.x * GEMV_ROWS;

    uint32_t expert = 0, total_pairs = 0;
    const uint32_t *pair_src = nullptr;  // routed mode: sorted pairs of this expert
    if (!route_prologue<FUSED>(P, ids_s, first_s, &expert_s, &npairs_s, row0, GEMV_ROWS, expert,
                               total_pairs, pair_src))
        return;

    if constexpr (KIND == K_CB2 || KIND == K_CB3 || KIND == K_CB4) {
        if (tid < (1u << kind_bits(KIND)))
            cb_s[tid] = f16_bits_to_f32(__ldg((const unsigned short *)P.aux + tid));
    }

    const uint32_t warp = tid >> 5, lane = tid & 31u;
    const uint32_t rsub = lane / GEMV_LPR, l8 = lane % GEMV_LPR;
    const uint32_t row = row0 + warp * (32 / GEMV_LPR) + rsub;  // logical row (glu_row)
    const bool row_ok = row < P.n;
    const uint32_t row_c = glu_row(row_ok ? row : P.n - 1, P.glu_nh);  // weight row; clamped loads stay in bounds
    constexpr bool AFF = (KIND == K_AFF4 || KIND == K_AFF6 || KIND == K_AFF8);
    // the expert's packed rows, scales and (affine) biases: slices of the contiguous
    // arrays, or the expert's own buffers from the pointer tables
    const uint8_t *wbase, *sbase, *bbase;
    size_t row_index = (size_t)expert * P.n + row_c;
    int load_mode = P.load_mode;
    if (P.packed_ptrs) {
        wbase = (const uint8_t *)__ldg(P.packed_ptrs + expert);
        if (!wbase) return;  // expert held elsewhere: its pairs' rows are not ours to write
        sbase = (const uint8_t *)__ldg(P.scale_ptrs + expert);
        bbase = AFF ? (const uint8_t *)__ldg(P.bias_ptrs + expert) : nullptr;
        const uintptr_t sa = (uintptr_t)sbase | (AFF ? (uintptr_t)bbase : 0u);
        if (!sbase || (AFF && !bbase) || (KIND != K_NVFP4 && KIND != K_MXFP4 && (sa & 1u))) {
            // scales / biases missing or not 2-byte aligned: skip the expert, flag it
            if (tid == 0 && blockIdx.x == 0) atomicOr(P.err, ERR_BAD_POINTER);
            return;
        }
        row_index = row_c;
        const uintptr_t wa = (uintptr_t)wbase;
        load_mode = (wa % 16u == 0 && P.row_bytes % 16u == 0) ? 16 : (wa % 4u == 0 && P.row_bytes % 4u == 0) ? 4 : 1;
    } else {
        wbase = P.packed;
        sbase = (const uint8_t *)P.scales;
        bbase = (const uint8_t *)P.aux;
    }

    GemvCtx c;
    c.row = wbase + row_index * P.row_bytes;
    c.row_bytes = P.row_bytes;
    c.gs = P.gs;
    c.groups = P.groups;
    c.codebook = (const uint16_t *)P.aux;
    if constexpr (KIND == K_NVFP4 || KIND == K_MXFP4) {  // byte scales
        c.scales = (const uint8_t *)sbase + row_index * P.groups;
        c.biases = nullptr;
    } else {
        c.scales = (const uint16_t *)sbase + row_index * P.groups;
        c.biases = AFF ? (const void *)((const uint16_t *)bbase + row_index * P.groups) : nullptr;
    }
    const float s2 = (KIND == K_NVFP4) ? __ldg((const float *)P.aux + expert) : 1.f;

    for (uint32_t pb = 0; pb < total_pairs; pb += NPB) {
        const uint32_t np = tmin<uint32_t>(NPB, total_pairs - pb);
        __syncthreads();  // previous batch's x reads are done
        load_pairs<FUSED>(P, ids_s, expert, pair_src, pb, np, pairs_s);
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
                    load_unit<U::UW>(c.row, u, c.row_bytes, load_mode, w[ub]);
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
        const float bv = load_bias(P.bias, P.bias_dtype, (size_t)expert * P.n + row_c);
        if (P.glu_nh) {
            // gate rows sit in even row slots, the matching up row GEMV_LPR lanes further on
#pragma unroll
            for (int q = 0; q < NPB; q++) {
                const float y = acc[q] * s2 + bv;
                const float up = __shfl_xor_sync(0xFFFFFFFFu, y, GEMV_LPR);
                if (l8 == 0 && row_ok && !(rsub & 1u) && (uint32_t)q < np)
                    store_out(P.out, P.out_dtype, (size_t)pairs_s[q] * P.glu_nh + (row >> 1),
                              glu_act(P.act, y) * up);
            }
        } else if (l8 == 0 && row_ok) {
#pragma unroll
            for (int q = 0; q < NPB; q++)
                if ((uint32_t)q < np)
                    store_out(P.out, P.out_dtype, (size_t)pairs_s[q] * P.n + row, acc[q] * s2 + bv);
        }
    }
}


// ----------------------------------------------------------- 4-bit affine, DP4A
//
// Exact integer dot products for 4-bit affine weights. For each 32-code unit u
// of x (one 16-byte load of a weight row), x is written once per CTA as a
// 24-bit fixed-point integer q_j = rint(x_j * 2^-E_u), E_u chosen from the
// unit's largest |x| so that |q_j| < 2^23, and split into three byte planes
// (q = b2*2^16 + b1*2^8 + b0, b0/b1 unsigned, b2 signed). Then
//     sum_j c_j x_j = 2^E_u * (sum c_j b0_j + 2^8 sum c_j b1_j + 2^16 sum c_j b2_j)
// where each inner sum is exact in int32 and computed four codes per dp4a. The
// group factorisation sum_j (c_j s + b) x_j = s * sum_j c_j x_j + b * sum_j x_j
// needs one fp32 FMA pair per unit. The only roundings are q_j (below 2^-23
// of the unit's largest |x|) and the fp32 combination of the partial sums.
// Weight rows are streamed once with 16-byte non-allocating loads issued
// before the x planes and scales are staged.
constexpr int DP_UMAX = 12;  // 16-byte units per lane per pass
constexpr int DP_PW = 28;    // u32 words of x planes per unit (24 used; 28 keeps LDS.128 conflict-free)

__device__ __forceinline__ uint32_t dp4a_uu(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("dp4a.u32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

__device__ __forceinline__ int32_t dp4a_us(uint32_t a, uint32_t b, int32_t c) {
    int32_t d;
    asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

__device__ __forceinline__ uint4 ldg_stream16(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ void sts8(uint32_t addr, uint32_t v) {
    asm volatile("st.shared.u8 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

template <int NPB>
__device__ __forceinline__ void dp4a_unit(const uint4 w, const uint32_t *planes_u, uint32_t plane_stride,
                                          const float *uscale_u, const float *usum_u,
                                          uint32_t sum_stride, float s, float b, float (&acc)[NPB]) {
    const uint32_t lo0 = w.x & 0x0F0F0F0Fu, hi0 = (w.x >> 4) & 0x0F0F0F0Fu;
    const uint32_t lo1 = w.y & 0x0F0F0F0Fu, hi1 = (w.y >> 4) & 0x0F0F0F0Fu;
    const uint32_t lo2 = w.z & 0x0F0F0F0Fu, hi2 = (w.z >> 4) & 0x0F0F0F0Fu;
    const uint32_t lo3 = w.w & 0x0F0F0F0Fu, hi3 = (w.w >> 4) & 0x0F0F0F0Fu;
#pragma unroll
    for (int q = 0; q < NPB; q++) {
        const uint4 *pl = (const uint4 *)(planes_u + q * plane_stride);
        const uint4 v0 = pl[0], v1 = pl[1], v2 = pl[2], v3 = pl[3], v4 = pl[4], v5 = pl[5];
        // plane words per unit: [word][plane][lo/hi]
        uint32_t a0 = dp4a_uu(lo0, v0.x, 0u);
        a0 = dp4a_uu(hi0, v0.y, a0);
        uint32_t a1 = dp4a_uu(lo0, v0.z, 0u);
        a1 = dp4a_uu(hi0, v0.w, a1);
        int32_t a2 = dp4a_us(lo0, v1.x, 0);
        a2 = dp4a_us(hi0, v1.y, a2);
        a0 = dp4a_uu(lo1, v1.z, a0);
        a0 = dp4a_uu(hi1, v1.w, a0);
        a1 = dp4a_uu(lo1, v2.x, a1);
        a1 = dp4a_uu(hi1, v2.y, a1);
        a2 = dp4a_us(lo1, v2.z, a2);
        a2 = dp4a_us(hi1, v2.w, a2);
        a0 = dp4a_uu(lo2, v3.x, a0);
        a0 = dp4a_uu(hi2, v3.y, a0);
        a1 = dp4a_uu(lo2, v3.z, a1);
        a1 = dp4a_uu(hi2, v3.w, a1);
        a2 = dp4a_us(lo2, v4.x, a2);
        a2 = dp4a_us(hi2, v4.y, a2);
        a0 = dp4a_uu(lo3, v4.z, a0);
        a0 = dp4a_uu(hi3, v4.w, a0);
        a1 = dp4a_uu(lo3, v5.x, a1);
        a1 = dp4a_uu(hi3, v5.y, a1);
        a2 = dp4a_us(lo3, v5.z, a2);
        a2 = dp4a_us(hi3, v5.w, a2);
        const float d = fmaf((float)a2, 65536.f, fmaf((float)a1, 256.f, (float)a0));
        acc[q] = fmaf(s, d * uscale_u[q * sum_stride], fmaf(b, usum_u[q * sum_stride], acc[q]));
    }
}

template <int NPB, bool FUSED>
__global__ void __launch_bounds__(GEMV_THREADS)
gemv_aff4_dp4a(const GemvParams P) {
    extern __shared__ __align__(16) uint32_t dsm[];
    __shared__ uint32_t ids_s[FUSED_MAX_R];
    __shared__ uint32_t first_s[FUSED_MAX_R];
    __shared__ uint32_t pairs_s[NPB];
    __shared__ uint32_t expert_s, npairs_s;

    const uint32_t tid = threadIdx.x;
    const uint32_t row0 = blockIdx.x * GEMV_ROWS;
    uint32_t expert = 0, total_pairs = 0;
    const uint32_t *pair_src = nullptr;
    if (!route_prologue<FUSED>(P, ids_s, first_s, &expert_s, &npairs_s, row0, GEMV_ROWS, expert,
                               total_pairs, pair_src))
        return;

    const uint32_t nu = P.n_units;  // 16-byte units (32 codes) per row
    const uint32_t G = P.groups;
    uint32_t *planes = dsm;                                          // [NPB][nu][DP_PW]
    float *uscale = (float *)(planes + (size_t)NPB * nu * DP_PW);    // [NPB][nu]
    float *usum = uscale + NPB * nu;                                 // [NPB][nu]
    uint32_t *sb = (uint32_t *)(usum + NPB * nu);                    // [GEMV_ROWS][G]

    const uint32_t warp = tid >> 5, lane = tid & 31u;
    const uint32_t rsub = lane / GEMV_LPR, l8 = lane % GEMV_LPR;
    const uint32_t rloc = warp * (32 / GEMV_LPR) + rsub;
    const uint32_t row = row0 + rloc;
    const bool row_ok = row < P.n;
    const size_t row_index = (size_t)expert * P.n + (row_ok ? row : P.n - 1);
    const uint8_t *rowp = P.packed + row_index * P.row_bytes;
    const uint32_t upg = P.gs / 32u;  // units per group

    for (uint32_t pb = 0; pb < total_pairs; pb += NPB) {
        const uint32_t np = tmin<uint32_t>(NPB, total_pairs - pb);
        float acc[NPB];
#pragma unroll
        for (int q = 0; q < NPB; q++) acc[q] = 0.f;
        for (uint32_t base = 0; base < nu; base += GEMV_LPR * DP_UMAX) {
            uint4 w[DP_UMAX];
#pragma unroll
            for (int i = 0; i < DP_UMAX; i++) {
                const uint32_t u = base + l8 + GEMV_LPR * i;
                w[i] = u < nu ? ldg_stream16(rowp + 16u * u) : make_uint4(0, 0, 0, 0);
            }
            if (base == 0) {
                __syncthreads();  // previous batch's planes are no longer read
                load_pairs<FUSED>(P, ids_s, expert, pair_src, pb, np, pairs_s);
                if (pb == 0) {
                    // scales and biases of this CTA's rows, packed (bf16 scale | bf16 bias << 16)
                    const size_t sbase = ((size_t)expert * P.n + row0) * G;
                    const uint32_t nrows = tmin<uint32_t>(GEMV_ROWS, P.n - row0);
                    const unsigned short *sc = (const unsigned short *)P.scales + sbase;
                    const unsigned short *bi = (const unsigned short *)P.aux + sbase;
                    for (uint32_t idx = tid; idx < nrows * G; idx += blockDim.x)
                        sb[idx] = (uint32_t)__ldg(sc + idx) | ((uint32_t)__ldg(bi + idx) << 16);
                }
                __syncthreads();
                // x planes, one warp per (pair, unit), lane = code within the unit
                const uint32_t plane_base = ptx_smem_addr(planes);
                for (uint32_t idx = warp; idx < NPB * nu; idx += GEMV_THREADS / 32) {
                    const uint32_t q = idx / nu, u = idx - q * nu;
                    const uint32_t j = u * 32u + lane;
                    float x = 0.f;
                    if (q < np && j < P.k) {
                        const uint32_t t = pairs_s[q] / P.n_expert_used;
                        x = load_x(P.x, P.x_dtype, (size_t)t * P.k + j);
                    }
                    const uint32_t eb = (__float_as_uint(x) >> 23) & 0xFFu;
                    const uint32_t emax = __reduce_max_sync(0xFFFFFFFFu, eb);
                    int E = (int)emax - 149;
                    E = E < -126 ? -126 : E;
                    const float inv = __uint_as_float((uint32_t)(127 - E) << 23);  // 2^-E
                    // |x * 2^-E| < 2^23; the clamp keeps a value rounded up to 2^23 in the planes
                    const int qv = max(-0x7FFFFF, min(0x7FFFFF, __float2int_rn(x * inv)));
                    const uint32_t wd = lane >> 3, nib = lane & 7u;
                    const uint32_t off = plane_base + (idx * DP_PW) * 4u +
                                         ((wd * 3u) * 2u + (nib & 1u)) * 4u + (nib >> 1);
                    sts8(off, (uint32_t)qv & 0xFFu);
                    sts8(off + 8u, ((uint32_t)qv >> 8) & 0xFFu);
                    sts8(off + 16u, ((uint32_t)qv >> 16) & 0xFFu);
                    float sum = x;
#pragma unroll
                    for (int d = 16; d > 0; d >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, d);
                    if (lane == 0) {
                        uscale[idx] = __uint_as_float((uint32_t)(127 + E) << 23);  // 2^E
                        usum[idx] = sum;
                    }
                }
                __syncthreads();
            }
#pragma unroll
            for (int i = 0; i < DP_UMAX; i++) {
                const uint32_t u = base + l8 + GEMV_LPR * i;
                if (u < nu) {
                    const uint32_t g = tmin<uint32_t>(u / upg, G - 1u);
                    const uint32_t sbv = sb[rloc * G + g];
                    dp4a_unit<NPB>(w[i], planes + u * DP_PW, nu * DP_PW, uscale + u, usum + u, nu,
                                   bf16_bits_to_f32(sbv & 0xFFFFu), bf16_bits_to_f32(sbv >> 16),
                                   acc);
                }
            }
        }
#pragma unroll
        for (int q = 0; q < NPB; q++) {
#pragma unroll
            for (int d = GEMV_LPR / 2; d > 0; d >>= 1) acc[q] += __shfl_xor_sync(0xFFFFFFFFu, acc[q], d);
        }
        if (l8 == 0 && row_ok) {
            const float bv = load_bias(P.bias, P.bias_dtype, (size_t)expert * P.n + row);
#pragma unroll
            for (int q = 0; q < NPB; q++)
                if ((uint32_t)q < np) store_out(P.out, P.out_dtype, (size_t)pairs_s[q] * P.n + row, acc[q] + bv);
        }
    }
}

size_t dp4a_smem(const GemvParams &P, int npb) {
    return (size_t)npb * P.n_units * (DP_PW + 2) * 4 + (size_t)GEMV_ROWS * P.groups * 4;
}

template <int NPB, bool FUSED>
cudaError_t launch_dp4a_one(const GemvParams &P, dim3 grid, cudaStream_t st) {
    const size_t smem = dp4a_smem(P, NPB);
    auto kern = gemv_aff4_dp4a<NPB, FUSED>;
    if (smem > 48 * 1024) {
        static int smem_set[64];
        cudaError_t e = ensure_dyn_smem(kern, smem, smem_set);
        if (e != cudaSuccess) return e;
    }
    kern<<<grid, GEMV_THREADS, smem, st>>>(P);
    return cudaGetLastError();
}

template <bool FUSED>
cudaError_t launch_dp4a(const GemvParams &P, uint32_t npb, dim3 grid, cudaStream_t st) {
    while (npb > 1 && dp4a_smem(P, (int)npb) > GEMV_SMEM_BUDGET) npb >>= 1;
    if (npb <= 1) return launch_dp4a_one<1, FUSED>(P, grid, st);
    if (npb <= 2) return launch_dp4a_one<2, FUSED>(P, grid, st);
    if (npb <= 4) return launch_dp4a_one<4, FUSED>(P, grid, st);
    return launch_dp4a_one<8, FUSED>(P, grid, st);
}

// The DP4A kernel covers 4-bit affine rows of whole 16-byte units with groups of
// whole 32-code units.
bool dp4a_ok(const QmmArgs &a) {
    return a.kind == K_AFF4 && a.group_size % 32 == 0 && a.row_bytes % 16 == 0 &&
           (uintptr_t)a.packed % 16 == 0 &&
           (size_t)GEMV_ROWS * a.groups * 4 + (size_t)(a.row_bytes / 16) * (DP_PW + 2) * 4 <= GEMV_SMEM_BUDGET;
}


// ------------------------------------------ 4-bit affine, DP4A, TMA-staged rows
//
// Same arithmetic as gemv_aff4_dp4a, but each warp's weight rows (contiguous
// in memory: rows of one expert are adjacent) arrive by one bulk TMA copy into
// shared memory, signalled on that warp's mbarrier, and x arrives the same way
// (for calls with few tokens, before the expert is even known). 512 threads per
// CTA; LPR lanes per row, so a CTA holds 512/LPR rows and each lane a handful of
// 16-byte units, which keeps a decode call's CTAs resident in one wave.
// Modes: PAIR (one CTA column per pair, no deduplication: the m = 1 case),
// FUSED (distinct experts ranked in the CTA, R <= 64), ROUTED (routing prologue).
enum { MODE_PAIR = 0, MODE_FUSED = 1, MODE_ROUTED = 2 };
constexpr int TMA_THREADS = 512;
constexpr int TMA_WARPS = TMA_THREADS / 32;

struct TmaLayout {
    uint32_t w, xraw, planes, uscale, usum, sc, bi, total;
};

__host__ __device__ inline uint32_t al16u(uint32_t v) { return (v + 15u) & ~15u; }

__host__ __device__ inline TmaLayout tma_layout(uint32_t rb, uint32_t row_bytes, uint32_t xraw_bytes,
                                                uint32_t npb, uint32_t nu, uint32_t G) {
    TmaLayout L;
    L.w = 0;
    L.xraw = al16u(rb * row_bytes);
    L.planes = al16u(L.xraw + xraw_bytes);
    L.uscale = L.planes + npb * nu * DP_PW * 4u;
    L.usum = L.uscale + npb * nu * 4u;
    L.sc = al16u(L.usum + npb * nu * 4u);
    L.bi = al16u(L.sc + rb * G * 2u);
    L.total = al16u(L.bi + rb * G * 2u);
    return L;
}

// Eight consecutive x values (16-byte aligned) from a shared-memory row.
__device__ __forceinline__ void smem_x8(const uint8_t *xr, int dt, uint32_t idx, float (&v)[8]) {
    if (dt == DT_F32) {
        const float4 a = *(const float4 *)(xr + 4u * idx), b = *(const float4 *)(xr + 4u * idx + 16u);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    } else {
        const uint4 h = *(const uint4 *)(xr + 2u * idx);
        const uint32_t hw[4] = {h.x, h.y, h.z, h.w};
#pragma unroll
        for (int i = 0; i < 4; i++) {
            if (dt == DT_BF16) {
                v[2 * i] = __uint_as_float(hw[i] << 16);
                v[2 * i + 1] = __uint_as_float(hw[i] & 0xFFFF0000u);
            } else {
                v[2 * i] = f16_bits_to_f32(hw[i] & 0xFFFFu);
                v[2 * i + 1] = f16_bits_to_f32(hw[i] >> 16);
            }
        }
    }
}

// Build the x planes of one 8-code word (lanes 4k..4k+3 of a warp hold the four
// words of one unit). All 32 lanes must call it.
__device__ __forceinline__ void plane_word(const float (&v)[8], uint32_t *unit_planes, uint32_t wd,
                                           float *uscale_u, float *usum_u, bool store) {
    uint32_t eb = 0;
#pragma unroll
    for (int i = 0; i < 8; i++) eb = max(eb, (__float_as_uint(v[i]) >> 23) & 0xFFu);
    eb = max(eb, __shfl_xor_sync(0xFFFFFFFFu, eb, 1));
    eb = max(eb, __shfl_xor_sync(0xFFFFFFFFu, eb, 2));
    int E = (int)eb - 149;
    E = E < -126 ? -126 : E;
    const float inv = __uint_as_float((uint32_t)(127 - E) << 23);  // 2^-E, |x * 2^-E| < 2^23
    int q[8];
#pragma unroll
    for (int i = 0; i < 8; i++) q[i] = max(-0x7FFFFF, min(0x7FFFFF, __float2int_rn(v[i] * inv)));  // < 2^23
    uint32_t pw[6];
#pragma unroll
    for (int p = 0; p < 3; p++) {
        // lo word: bytes p of q0, q2, q4, q6; hi word: bytes p of q1, q3, q5, q7
        const uint32_t sel = (uint32_t)p | ((uint32_t)(4 + p) << 4);
        const uint32_t l01 = __byte_perm((uint32_t)q[0], (uint32_t)q[2], sel);
        const uint32_t l23 = __byte_perm((uint32_t)q[4], (uint32_t)q[6], sel);
        const uint32_t h01 = __byte_perm((uint32_t)q[1], (uint32_t)q[3], sel);
        const uint32_t h23 = __byte_perm((uint32_t)q[5], (uint32_t)q[7], sel);
        pw[2 * p] = __byte_perm(l01, l23, 0x5410);
        pw[2 * p + 1] = __byte_perm(h01, h23, 0x5410);
    }
    if (store) {
        uint2 *dst = (uint2 *)(unit_planes + wd * 6u);  // [word][plane][lo/hi]
        dst[0] = make_uint2(pw[0], pw[1]);
        dst[1] = make_uint2(pw[2], pw[3]);
        dst[2] = make_uint2(pw[4], pw[5]);
    }
    float sum = ((v[0] + v[1]) + (v[2] + v[3])) + ((v[4] + v[5]) + (v[6] + v[7]));
    sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 1);
    sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 2);
    if (store && wd == 0) {
        *uscale_u = __uint_as_float((uint32_t)(127 + E) << 23);  // 2^E
        *usum_u = sum;
    }
}

template <int NPB, int MODE, int LPR>
__global__ void __launch_bounds__(TMA_THREADS)
gemv_aff4_tma(const GemvParams P) {
    constexpr uint32_t RB = TMA_THREADS / LPR;  // rows per CTA
    constexpr uint32_t RPW = 32 / LPR;          // rows per warp
    constexpr uint64_t WAIT = 1000000000ull;
    extern __shared__ __align__(128) uint8_t dsm8[];
    __shared__ uint32_t ids_s[FUSED_MAX_R];
    __shared__ uint32_t first_s[FUSED_MAX_R];
    __shared__ uint32_t pairs_s[NPB];
    __shared__ uint32_t expert_s, npairs_s;
    __shared__ __align__(8) uint64_t bar_w[TMA_WARPS];
    __shared__ __align__(8) uint64_t bar_x, bar_s;
    __shared__ int abort_s;

    const uint32_t tid = threadIdx.x, warp = tid >> 5, lane = tid & 31u;
    const uint32_t row0 = blockIdx.x * RB;
    const uint32_t nu = P.n_units, G = P.groups, rbytes = P.row_bytes;
    const uint32_t xsz = P.x_dtype == DT_F32 ? 4u : 2u;
    const uint32_t xrow = P.k * xsz;
    const bool spec = MODE != MODE_ROUTED && P.x_spec;  // all m x rows staged up front
    const TmaLayout L = tma_layout(RB, rbytes, spec ? P.m * xrow : NPB * xrow, NPB, nu, G);
    const uint32_t sbase = ptx::smem_u32(dsm8);
    volatile int *abort_flag = &abort_s;

    if (tid == 0) {
        for (int i = 0; i < TMA_WARPS; i++) ptx::mbar_init(ptx::smem_u32(&bar_w[i]), 1);
        ptx::mbar_init(ptx::smem_u32(&bar_x), 1);
        ptx::mbar_init(ptx::smem_u32(&bar_s), 1);
        ptx::fence_mbar_init();
        abort_s = 0;
    }
    __syncthreads();
    const uint32_t bx = ptx::smem_u32(&bar_x), bs = ptx::smem_u32(&bar_s);
    if (spec && tid == 0) {
        ptx::mbar_arrive_expect_tx(bx, P.m * xrow);
        ptx::bulk_g2s(sbase + L.xraw, P.x, P.m * xrow, bx);
    }

    uint32_t expert = 0, total_pairs = 0;
    const uint32_t *pair_src = nullptr;
    bool work;
    if constexpr (MODE == MODE_PAIR) {
        const uint32_t p = blockIdx.y;
        expert = __ldg(P.ids + p);
        work = expert < P.num_experts;
        total_pairs = 1;
        if (!work) {
            // out-of-range id: zero this pair's rows of the block
            for (uint32_t r = row0 + tid; r < tmin<uint32_t>(row0 + RB, P.n); r += blockDim.x)
                store_out(P.out, P.out_dtype, (size_t)p * P.n + r, 0.f);
            if (blockIdx.x == 0 && tid == 0) atomicOr(P.err, ERR_BAD_ID);
        }
    } else {
        work = route_prologue<MODE == MODE_FUSED>(P, ids_s, first_s, &expert_s, &npairs_s, row0, RB,
                                                  expert, total_pairs, pair_src);
    }
    if (!work) {
        if (spec) ptx::mbar_wait_bounded(bx, 0, nullptr, P.err, ERR_TIMEOUT, WAIT);  // drain the copy
        return;
    }

    // scales and biases of the CTA's rows (bf16), by bulk copy when aligned
    const uint32_t nrows = tmin<uint32_t>(RB, P.n - row0);
    const size_t soff = ((size_t)expert * P.n + row0) * G;
    const uint32_t sbytes = nrows * G * 2u;
    const bool s_bulk = (soff * 2u) % 16u == 0 && sbytes % 16u == 0 &&
                        (uintptr_t)P.scales % 16u == 0 && (uintptr_t)P.aux % 16u == 0;
    if (s_bulk) {
        if (tid == 0) {
            ptx::mbar_arrive_expect_tx(bs, 2u * sbytes);
            ptx::bulk_g2s(sbase + L.sc, (const unsigned short *)P.scales + soff, sbytes, bs);
            ptx::bulk_g2s(sbase + L.bi, (const unsigned short *)P.aux + soff, sbytes, bs);
        }
    } else {
        unsigned short *sc = (unsigned short *)(dsm8 + L.sc), *bi = (unsigned short *)(dsm8 + L.bi);
        for (uint32_t idx = tid; idx < nrows * G; idx += blockDim.x) {
            sc[idx] = __ldg((const unsigned short *)P.scales + soff + idx);
            bi[idx] = __ldg((const unsigned short *)P.aux + soff + idx);
        }
    }

    // weight rows of this warp: one bulk copy
    if (lane == 0) {
        const uint32_t rb0 = row0 + warp * RPW;
        const uint32_t nr = rb0 < P.n ? tmin<uint32_t>(RPW, P.n - rb0) : 0u;
        const uint32_t bw = ptx::smem_u32(&bar_w[warp]);
        if (nr) {
            ptx::mbar_arrive_expect_tx(bw, nr * rbytes);
            ptx::bulk_g2s(sbase + L.w + warp * RPW * rbytes,
                          P.packed + ((size_t)expert * P.n + rb0) * rbytes, nr * rbytes, bw);
        } else {
            ptx::mbar_arrive(bw);
        }
    }
    uint32_t *planes = (uint32_t *)(dsm8 + L.planes);
    float *uscale = (float *)(dsm8 + L.uscale);
    float *usum = (float *)(dsm8 + L.usum);
    const unsigned short *sc = (const unsigned short *)(dsm8 + L.sc);
    const unsigned short *bi = (const unsigned short *)(dsm8 + L.bi);
    const uint32_t rloc = warp * RPW + lane / LPR, l = lane % LPR;
    const uint32_t row = row0 + rloc;
    const uint8_t *wrow = dsm8 + L.w + rloc * rbytes;
    const uint32_t upg = P.gs / 32u;
    const uint32_t nwords = nu * 4u;  // 8-code words per x row
    uint32_t batch = 0;

    for (uint32_t pb = 0; pb < total_pairs; pb += NPB, batch++) {
        const uint32_t np = tmin<uint32_t>(NPB, total_pairs - pb);
        if (pb > 0) __syncthreads();  // planes of the previous batch are no longer read
        if constexpr (MODE == MODE_PAIR) {
            if (tid == 0) pairs_s[0] = blockIdx.y;
        } else {
            load_pairs<MODE == MODE_FUSED>(P, ids_s, expert, pair_src, pb, np, pairs_s);
        }
        __syncthreads();
        if (!spec && tid == 0) {
            ptx::mbar_arrive_expect_tx(bx, np * xrow);
            for (uint32_t q = 0; q < np; q++)
                ptx::bulk_g2s(sbase + L.xraw + q * xrow,
                              (const uint8_t *)P.x + (size_t)(pairs_s[q] / P.n_expert_used) * xrow,
                              xrow, bx);
        }
        const bool x_ok = ptx::mbar_wait_bounded(bx, spec ? 0u : (batch & 1u), abort_flag, P.err,
                                                 ERR_TIMEOUT, WAIT);
        // x planes: one thread per (pair, 8-code word); 4 consecutive lanes hold a unit
        if (__all_sync(0xFFFFFFFFu, x_ok)) {
            for (uint32_t base = warp * 32u; base < NPB * nwords; base += TMA_THREADS) {
                const uint32_t idx = base + lane;
                float v[8];
                const uint32_t q = idx / nwords, r = idx - q * nwords;
                const uint32_t u = r >> 2, wd = r & 3u;
                const uint32_t j = u * 32u + wd * 8u;
                const bool valid = idx < NPB * nwords;
                if (valid && q < np && j < P.k) {
                    const uint32_t xr = spec ? pairs_s[q] / P.n_expert_used : q;
                    smem_x8(dsm8 + L.xraw, P.x_dtype, xr * P.k + j, v);
#pragma unroll
                    for (int i = 0; i < 8; i++)
                        if (j + i >= P.k) v[i] = 0.f;  // codes past k meet x = 0
                } else {
#pragma unroll
                    for (int i = 0; i < 8; i++) v[i] = 0.f;
                }
                const uint32_t uidx = valid ? q * nu + u : 0u;
                plane_word(v, planes + uidx * DP_PW, wd, uscale + uidx, usum + uidx, valid);
            }
        }
        bool s_ok = true;
        if (pb == 0 && s_bulk) s_ok = ptx::mbar_wait_bounded(bs, 0, abort_flag, P.err, ERR_TIMEOUT, WAIT);
        __syncthreads();
        bool w_ok = true;
        if (pb == 0)
            w_ok = ptx::mbar_wait_bounded(ptx::smem_u32(&bar_w[warp]), 0, abort_flag, P.err,
                                          ERR_TIMEOUT, WAIT);
        // a wait that gave up has flagged ERR_TIMEOUT; the warp then skips its work but
        // keeps the block's barrier sequence
        if (!__all_sync(0xFFFFFFFFu, x_ok && s_ok && w_ok && !*abort_flag)) continue;

        float acc[NPB], acc2[NPB];
#pragma unroll
        for (int q = 0; q < NPB; q++) acc[q] = acc2[q] = 0.f;
        uint32_t u = l;
        for (; u + LPR < nu; u += 2 * LPR) {  // two independent units per step
            const uint4 w0 = *(const uint4 *)(wrow + 16u * u);
            const uint4 w1 = *(const uint4 *)(wrow + 16u * (u + LPR));
            const uint32_t si0 = rloc * G + tmin<uint32_t>(u / upg, G - 1u);
            const uint32_t si1 = rloc * G + tmin<uint32_t>((u + LPR) / upg, G - 1u);
            dp4a_unit<NPB>(w0, planes + u * DP_PW, nu * DP_PW, uscale + u, usum + u, nu,
                           bf16_bits_to_f32(sc[si0]), bf16_bits_to_f32(bi[si0]), acc);
            dp4a_unit<NPB>(w1, planes + (u + LPR) * DP_PW, nu * DP_PW, uscale + u + LPR,
                           usum + u + LPR, nu, bf16_bits_to_f32(sc[si1]), bf16_bits_to_f32(bi[si1]),
                           acc2);
        }
        if (u < nu) {
            const uint4 w0 = *(const uint4 *)(wrow + 16u * u);
            const uint32_t si0 = rloc * G + tmin<uint32_t>(u / upg, G - 1u);
            dp4a_unit<NPB>(w0, planes + u * DP_PW, nu * DP_PW, uscale + u, usum + u, nu,
                           bf16_bits_to_f32(sc[si0]), bf16_bits_to_f32(bi[si0]), acc);
        }
#pragma unroll
        for (int q = 0; q < NPB; q++) {
            acc[q] += acc2[q];
#pragma unroll
            for (int d = LPR / 2; d > 0; d >>= 1) acc[q] += __shfl_xor_sync(0xFFFFFFFFu, acc[q], d);
        }
        if (l == 0 && row < P.n) {
            const float bv = load_bias(P.bias, P.bias_dtype, (size_t)expert * P.n + row);
#pragma unroll
            for (int q = 0; q < NPB; q++)
                if ((uint32_t)q < np) store_out(P.out, P.out_dtype, (size_t)pairs_s[q] * P.n + row, acc[q] + bv);
        }
    }
    if (*abort_flag) {
        // a wait gave up: let this CTA's copies land before its shared memory is released
        ptx::mbar_wait_bounded(ptx::smem_u32(&bar_w[warp]), 0, nullptr, P.err, ERR_TIMEOUT, WAIT);
        ptx::mbar_wait_bounded(bx, spec ? 0u : ((batch - 1u) & 1u), nullptr, P.err, ERR_TIMEOUT, WAIT);
        if (s_bulk) ptx::mbar_wait_bounded(bs, 0, nullptr, P.err, ERR_TIMEOUT, WAIT);
    }
}

// Two-plane variant for the one-token kernel: x of a unit as 16-bit fixed point,
// q_j = rint(x_j * 2^-E_u) with |q_j| < 2^15 (clamped), split into an unsigned low
// byte plane and a signed high byte plane: q = b1 * 2^8 + b0. For bf16 and f16 x
// this is exact (x * 2^-E_u is then a multiple of 2^7 (bf16) or 2^4 (f16) below
// 2^15); for f32 x the rounding is below 2^-15 of the unit's largest |x|. Per word
// wd of the unit four plane words are stored: plane 0 lo, plane 0 hi, plane 1 lo,
// plane 1 hi (lo: bytes of codes 0, 2, 4, 6 of the word, hi: codes 1, 3, 5, 7).
constexpr int DP_PW2 = 20;  // u32 words per unit (16 used; 20 spreads the banks of per-lane loads)

__device__ __forceinline__ void plane_word2(const float (&v)[8], uint32_t *unit_planes, uint32_t wd,
                                            float *uscale_u, float *usum_u, bool store) {
    uint32_t eb = 0;
#pragma unroll
    for (int i = 0; i < 8; i++) eb = max(eb, (__float_as_uint(v[i]) >> 23) & 0xFFu);
    eb = max(eb, __shfl_xor_sync(0xFFFFFFFFu, eb, 1));
    eb = max(eb, __shfl_xor_sync(0xFFFFFFFFu, eb, 2));
    int E = (int)eb - 141;
    E = E < -126 ? -126 : E;
    const float inv = __uint_as_float((uint32_t)(127 - E) << 23);  // 2^-E, |x * 2^-E| < 2^15
    int q[8];
#pragma unroll
    for (int i = 0; i < 8; i++) q[i] = max(-0x7FFF, min(0x7FFF, __float2int_rn(v[i] * inv)));
    uint32_t pw[4];
#pragma unroll
    for (int p = 0; p < 2; p++) {
        const uint32_t sel = (uint32_t)p | ((uint32_t)(4 + p) << 4);
        const uint32_t l01 = __byte_perm((uint32_t)q[0], (uint32_t)q[2], sel);
        const uint32_t l23 = __byte_perm((uint32_t)q[4], (uint32_t)q[6], sel);
        const uint32_t h01 = __byte_perm((uint32_t)q[1], (uint32_t)q[3], sel);
        const uint32_t h23 = __byte_perm((uint32_t)q[5], (uint32_t)q[7], sel);
        pw[2 * p] = __byte_perm(l01, l23, 0x5410);
        pw[2 * p + 1] = __byte_perm(h01, h23, 0x5410);
    }
    if (store) *(uint4 *)(unit_planes + wd * 4u) = make_uint4(pw[0], pw[1], pw[2], pw[3]);
    float sum = ((v[0] + v[1]) + (v[2] + v[3])) + ((v[4] + v[5]) + (v[6] + v[7]));
    sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 1);
    sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 2);
    if (store && wd == 0) {
        *uscale_u = __uint_as_float((uint32_t)(127 + E) << 23);  // 2^E
        *usum_u = sum;
    }
}

// -------------------- 4-bit affine, one token: x planes held in registers
//
// With a single token every (token, slot) pair multiplies the same x row, so a
// lane can keep the x planes of its own slice of k in registers for every
// weight row it meets, and shared memory only carries the weight rows (each
// byte read once). Rows of all pairs are numbered globally (pair p's column c
// is row p*n + c) and split into equal contiguous ranges, two CTAs per SM, so
// every SM streams the same number of bytes whatever the experts. A group of
// LPR lanes owns one row at a time; lane l of the group holds 32-code units
// l, l+LPR, ..., UPL of them, as two byte planes of 16-bit fixed point
// (plane_word2, exact for bf16 and f16 x), so a 32-code unit takes 16 DP4A.
// Each warp's rows arrive by bulk copies (one per pair the range touches) on the
// warp's own mbarrier; scales, biases and x by bulk copies issued before the
// planes are built.
constexpr int ROWS_THREADS = 256;
constexpr int ROWS_WARPS = ROWS_THREADS / 32;
constexpr uint32_t ROWS_MAX_PAIRS = 64;

struct RowsLayout {
    uint32_t w, xraw, planes, uscale, usum, sc, bi, total;
};

__host__ __device__ inline RowsLayout rows_layout(uint32_t rb, uint32_t row_bytes, uint32_t x_bytes,
                                                  uint32_t nu, uint32_t G) {
    RowsLayout L;
    L.w = 0;
    L.xraw = al16u(rb * row_bytes);
    L.planes = al16u(L.xraw + x_bytes);
    L.uscale = L.planes + nu * DP_PW2 * 4u;
    L.usum = L.uscale + nu * 4u;
    L.sc = al16u(L.usum + nu * 4u);
    L.bi = al16u(L.sc + rb * G * 2u);
    L.total = al16u(L.bi + rb * G * 2u);
    return L;
}

// Integer dot product of one 32-code unit with two x planes held in registers
// (v[wd] = plane 0 lo, plane 0 hi, plane 1 lo, plane 1 hi of word wd): 16 DP4A in
// four chains. Each plane sum is below 2^17 in magnitude, so d = a0 + 2^8 a1 is
// exact in int32 and in fp32.
__device__ __forceinline__ float dp4a_unit_reg2(const uint4 w, const uint4 (&v)[4], float usc, float usm,
                                                float s, float b, float acc) {
    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
    uint32_t a0l = 0u, a0h = 0u;
    int32_t a1l = 0, a1h = 0;
#pragma unroll
    for (int i = 0; i < 4; i++) {
        const uint32_t lo = ww[i] & 0x0F0F0F0Fu, hi = (ww[i] >> 4) & 0x0F0F0F0Fu;
        a0l = dp4a_uu(lo, v[i].x, a0l);
        a0h = dp4a_uu(hi, v[i].y, a0h);
        a1l = dp4a_us(lo, v[i].z, a1l);
        a1h = dp4a_us(hi, v[i].w, a1h);
    }
    const float d = (float)((int32_t)(a0l + a0h) + ((a1l + a1h) << 8));
    return fmaf(s, d * usc, fmaf(b, usm, acc));
}

template <int LPR, int UPL, bool GLU>
__global__ void __launch_bounds__(ROWS_THREADS, 2)
gemv_aff4_rows(const GemvParams P, uint32_t rows_per_cta) {
    constexpr uint32_t RPI = 32 / LPR;  // rows a warp works on at once
    constexpr uint32_t AREAS = GLU ? 2u : 1u;
    constexpr uint64_t WAIT = 1000000000ull;
    extern __shared__ __align__(128) uint8_t dsm8[];
    __shared__ uint32_t ex_s[ROWS_MAX_PAIRS];
    __shared__ __align__(8) uint64_t bar_w[ROWS_WARPS];
    __shared__ __align__(8) uint64_t bar_x, bar_s, bar_never;
    __shared__ int abort_s;

    const uint32_t tid = threadIdx.x, warp = tid >> 5, lane = tid & 31u;
    // nn: rows of the walk per pair (with GLU one row of the walk is an output
    // element: gate row c in the first shared-memory area, up row n/2 + c in the second)
    const uint32_t n = P.n, nn = GLU ? P.glu_nh : n, nu = P.n_units, G = P.groups, rbytes = P.row_bytes;
    const uint32_t total_rows = P.R * nn;
    const uint32_t g0 = blockIdx.x * rows_per_cta;
    const uint32_t nrows = tmin<uint32_t>(rows_per_cta, total_rows - g0);
    const uint32_t p_first = g0 / nn, p_last = (g0 + nrows - 1u) / nn;
    const uint32_t xsz = P.x_dtype == DT_F32 ? 4u : 2u;
    const RowsLayout L = rows_layout(AREAS * rows_per_cta, rbytes, P.k * xsz, nu, G);
    const uint32_t sbase = ptx::smem_u32(dsm8);
    volatile int *abort_flag = &abort_s;
    const bool early = P.early_weights != 0;

    // a kernel launched after this one on the stream may be scheduled as soon as
    // SMs free up; it waits for this grid itself before touching what it writes
    ptx::griddep_launch_dependents();
    // programmatic launch: without early_weights every input may come from the
    // previous kernel on the stream, so wait for it first (a no-op otherwise)
    if (!early) ptx::griddep_wait();

    // experts of the pairs this CTA touches (loads in flight across the barrier)
    if (tid <= p_last - p_first) ex_s[tid] = __ldg(P.ids + p_first + tid);
    if (tid == 0) {
        for (int i = 0; i < ROWS_WARPS; i++) ptx::mbar_init(ptx::smem_u32(&bar_w[i]), 1);
        ptx::mbar_init(ptx::smem_u32(&bar_x), 1);
        ptx::mbar_init(ptx::smem_u32(&bar_s), 1);
        ptx::mbar_init(ptx::smem_u32(&bar_never), 1);  // completed by nothing
        ptx::fence_mbar_init();
        abort_s = 0;
    }
    __syncthreads();
    const uint32_t bx = ptx::smem_u32(&bar_x), bs = ptx::smem_u32(&bar_s);
    const uint32_t bw = ptx::smem_u32(&bar_w[warp]);
    if (tid == 0 && !early) {
        ptx::mbar_arrive_expect_tx(bx, P.k * xsz);
        ptx::bulk_g2s(sbase + L.xraw, P.x, P.k * xsz, bx);
    }
    // scales and biases of the CTA's rows: one bulk copy of each per pair and area when aligned
    const bool s_bulk = P.s_bulk != 0;
    if (s_bulk) {
        if (tid == 0) {
            uint32_t bytes = 0;
            for (uint32_t p = p_first; p <= p_last; p++) {
                const uint32_t lo = p == p_first ? g0 - p * nn : 0u;
                const uint32_t hi = p == p_last ? g0 + nrows - p * nn : nn;
                if (ex_s[p - p_first] < P.num_experts) bytes += AREAS * 2u * (hi - lo) * G * 2u;
            }
            ptx::mbar_arrive_expect_tx(bs, bytes);
            for (uint32_t p = p_first; p <= p_last; p++) {
                const uint32_t lo = p == p_first ? g0 - p * nn : 0u;
                const uint32_t hi = p == p_last ? g0 + nrows - p * nn : nn;
                const uint32_t e = ex_s[p - p_first];
                if (e >= P.num_experts) continue;
                for (uint32_t h = 0; h < AREAS; h++) {
                    const uint32_t dst = (h * rows_per_cta + p * nn + lo - g0) * G * 2u;
                    const size_t src = ((size_t)e * n + h * nn + lo) * G;
                    ptx::bulk_g2s(sbase + L.sc + dst, (const unsigned short *)P.scales + src, (hi - lo) * G * 2u, bs);
                    ptx::bulk_g2s(sbase + L.bi + dst, (const unsigned short *)P.aux + src, (hi - lo) * G * 2u, bs);
                }
            }
        }
    } else {
        unsigned short *sc = (unsigned short *)(dsm8 + L.sc), *bi = (unsigned short *)(dsm8 + L.bi);
        for (uint32_t h = 0; h < AREAS; h++) {
            for (uint32_t idx = tid; idx < nrows * G; idx += blockDim.x) {
                const uint32_t r = idx / G, gi = idx - r * G;
                const uint32_t g = g0 + r, p = g / nn, c = g - p * nn;
                const uint32_t e = ex_s[p - p_first];
                const size_t src = ((size_t)(e < P.num_experts ? e : 0u) * n + h * nn + c) * G + gi;
                sc[h * rows_per_cta * G + idx] = __ldg((const unsigned short *)P.scales + src);
                bi[h * rows_per_cta * G + idx] = __ldg((const unsigned short *)P.aux + src);
            }
        }
    }

    // this warp's rows [a, b) of the CTA's range, one bulk copy per pair (and area) they touch
    const uint32_t rpw = (nrows + ROWS_WARPS - 1) / ROWS_WARPS;
    const uint32_t a = tmin<uint32_t>(warp * rpw, nrows), b = tmin<uint32_t>(a + rpw, nrows);
    if (lane == 0) {
        uint32_t bytes = 0;
        for (uint32_t r = a; r < b;) {
            const uint32_t g = g0 + r, p = g / nn, c0 = g - p * nn;
            const uint32_t cnt = tmin<uint32_t>(b - r, nn - c0);
            const uint32_t e = ex_s[p - p_first];
            if (e < P.num_experts) bytes += AREAS * cnt * rbytes;
            r += cnt;
        }
        ptx::mbar_arrive_expect_tx(bw, bytes);
        for (uint32_t r = a; r < b;) {
            const uint32_t g = g0 + r, p = g / nn, c0 = g - p * nn;
            const uint32_t cnt = tmin<uint32_t>(b - r, nn - c0);
            const uint32_t e = ex_s[p - p_first];
            if (e < P.num_experts) {
                for (uint32_t h = 0; h < AREAS; h++)
                    ptx::bulk_g2s(sbase + L.w + (h * rows_per_cta + r) * rbytes,
                                  P.packed + ((size_t)e * n + h * nn + c0) * rbytes, cnt * rbytes, bw);
            } else if (c0 == 0) {
                atomicOr(P.err, ERR_BAD_ID);
            }
            r += cnt;
        }
    }
    if (early) {
        // ids, weights and scales were ready before the previous kernel began (the
        // caller's promise); x may be its output, and out may still be read by it
        ptx::griddep_wait();
        if (tid == 0) {
            ptx::mbar_arrive_expect_tx(bx, P.k * xsz);
            ptx::bulk_g2s(sbase + L.xraw, P.x, P.k * xsz, bx);
        }
    }
    // x planes, once per CTA: one thread per 8-code word, 4 consecutive lanes per unit
    uint32_t *planes = (uint32_t *)(dsm8 + L.planes);
    float *uscale = (float *)(dsm8 + L.uscale);
    float *usum = (float *)(dsm8 + L.usum);
    // failure-detection test hook: a wait nothing completes, so that the CTA aborts
    const bool f_ok = !P.fault_ns || warp != 0 ||
                      ptx::mbar_wait_bounded(ptx::smem_u32(&bar_never), 0, abort_flag, P.err, ERR_TIMEOUT,
                                             P.fault_ns);
    const bool x_ok = f_ok && ptx::mbar_wait_bounded(bx, 0, abort_flag, P.err, ERR_TIMEOUT, WAIT);
    if (__all_sync(0xFFFFFFFFu, x_ok)) {
        const uint32_t nwords = nu * 4u;
        for (uint32_t base = warp * 32u; base < nwords; base += ROWS_THREADS) {
            const uint32_t idx = base + lane;
            const bool valid = idx < nwords;
            const uint32_t u = valid ? idx >> 2 : 0u, wd = idx & 3u;
            const uint32_t j = u * 32u + wd * 8u;
            float v[8];
            if (valid && j < P.k) {
                smem_x8(dsm8 + L.xraw, P.x_dtype, j, v);
#pragma unroll
                for (int i = 0; i < 8; i++)
                    if (j + i >= P.k) v[i] = 0.f;  // codes past k meet x = 0
            } else {
#pragma unroll
                for (int i = 0; i < 8; i++) v[i] = 0.f;
            }
            plane_word2(v, planes + u * DP_PW2, wd, uscale + u, usum + u, valid);
        }
    }
    __syncthreads();

    // this lane's units and their planes, in registers for all its rows
    const uint32_t gi = lane / LPR, l = lane % LPR;
    const uint32_t upg = P.gs / 32u;
    uint4 pv[UPL][4];
    float usc[UPL], usm[UPL];
    uint32_t grp[UPL];
#pragma unroll
    for (int i = 0; i < UPL; i++) {
        const uint32_t u = tmin<uint32_t>(l + (uint32_t)i * LPR, nu - 1u);
        const uint4 *pl = (const uint4 *)(planes + u * DP_PW2);
#pragma unroll
        for (int t = 0; t < 4; t++) pv[i][t] = pl[t];
        usc[i] = uscale[u];
        usm[i] = usum[u];
        grp[i] = tmin<uint32_t>(u / upg, G - 1u);
    }
    bool s_ok = true;
    if (s_bulk) s_ok = ptx::mbar_wait_bounded(bs, 0, abort_flag, P.err, ERR_TIMEOUT, WAIT);
    const bool w_ok = ptx::mbar_wait_bounded(bw, 0, abort_flag, P.err, ERR_TIMEOUT, WAIT);
    if (!__all_sync(0xFFFFFFFFu, x_ok && s_ok && w_ok && !*abort_flag)) {
        // a wait gave up: let this warp's copies, the scale copies and the x copy land
        // before shared memory is released (each with the full limit)
        ptx::mbar_wait_bounded(bw, 0, nullptr, P.err, ERR_TIMEOUT, WAIT);
        if (s_bulk) ptx::mbar_wait_bounded(bs, 0, nullptr, P.err, ERR_TIMEOUT, WAIT);
        ptx::mbar_wait_bounded(bx, 0, nullptr, P.err, ERR_TIMEOUT, WAIT);
        return;
    }
    const unsigned short *sc = (const unsigned short *)(dsm8 + L.sc);
    const unsigned short *bi = (const unsigned short *)(dsm8 + L.bi);

    // rows a + gi, a + gi + RPI, ...: (pair, column) carried along
    uint32_t g = g0 + a + gi;
    uint32_t p = g / nn, c = g - p * nn;
    for (uint32_t r = a + gi; r < b + gi; r += RPI) {
        const bool valid = r < b;
        const uint32_t e = valid ? ex_s[p - p_first] : 0u;
        const bool live = valid && e < P.num_experts;
        float acc[AREAS];
#pragma unroll
        for (uint32_t h = 0; h < AREAS; h++) {
            acc[h] = 0.f;
            if (live) {
                const uint32_t rr = h * rows_per_cta + r;
                const uint8_t *wrow = dsm8 + L.w + rr * rbytes;
                const unsigned short *srow = sc + rr * G, *brow = bi + rr * G;
#pragma unroll
                for (int i = 0; i < UPL; i++) {
                    const uint32_t u = l + (uint32_t)i * LPR;
                    if (u < nu) {
                        const uint4 w = *(const uint4 *)(wrow + 16u * u);
                        acc[h] = dp4a_unit_reg2(w, pv[i], usc[i], usm[i], bf16_bits_to_f32(srow[grp[i]]),
                                                bf16_bits_to_f32(brow[grp[i]]), acc[h]);
                    }
                }
            }
#pragma unroll
            for (int d = LPR / 2; d > 0; d >>= 1) acc[h] += __shfl_xor_sync(0xFFFFFFFFu, acc[h], d);
        }
        if (valid && l == 0) {
            float v = 0.f;
            if (e < P.num_experts) {
                const size_t bb = (size_t)e * n + c;
                v = acc[0] + load_bias(P.bias, P.bias_dtype, bb);
                if constexpr (GLU) v = glu_act(P.act, v) * (acc[1] + load_bias(P.bias, P.bias_dtype, bb + nn));
            }
            store_out(P.out, P.out_dtype, (size_t)p * nn + c, v);
        }
        c += RPI;
        while (c >= nn) {  // pairs of fewer than RPI rows are stepped over whole
            c -= nn;
            p++;
        }
    }
}

// Lanes per row and units per lane for nu 32-code units: the pair with the
// fewest idle lanes, at most 3 units per lane (0 when nu is too large: the
// planes and two rows of units of 4 units per lane do not fit in registers).
void rows_shape(uint32_t nu, int *lpr, int *upl) {
    *lpr = 0;
    *upl = 0;
    double best = 0.0;
    for (int L = 32; L >= 4; L >>= 1) {
        const uint32_t U = (nu + L - 1) / L;
        if (U > 3 || U == 0) continue;
        const double eff = (double)nu / (double)(L * U);
        if (eff > best + 1e-9) {
            best = eff;
            *lpr = L;
            *upl = (int)U;
        }
    }
}

template <int LPR, int UPL, bool GLU>
cudaError_t launch_rows_t(const GemvParams &P, uint32_t rb, uint32_t ctas, size_t smem, cudaStream_t st) {
    auto kern = gemv_aff4_rows<LPR, UPL, GLU>;
    if (smem > 48 * 1024) {
        static int smem_set[64];
        cudaError_t e = ensure_dyn_smem(kern, smem, smem_set);
        if (e != cudaSuccess) return e;
    }
    if (!P.pdl) {
        kern<<<ctas, ROWS_THREADS, smem, st>>>(P, rb);
        return cudaGetLastError();
    }
    // programmatic dependent launch: may be scheduled before the previous kernel on
    // the stream completes; the kernel waits for it (griddepcontrol.wait) itself
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(ctas);
    cfg.blockDim = dim3(ROWS_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, P, rb);
}

template <int LPR>
cudaError_t launch_rows_l(const GemvParams &P, int upl, uint32_t rb, uint32_t ctas, size_t smem,
                          cudaStream_t st) {
    if (P.glu_nh) {
        switch (upl) {
            case 1: return launch_rows_t<LPR, 1, true>(P, rb, ctas, smem, st);
            case 2: return launch_rows_t<LPR, 2, true>(P, rb, ctas, smem, st);
            default: return launch_rows_t<LPR, 3, true>(P, rb, ctas, smem, st);
        }
    }
    switch (upl) {
        case 1: return launch_rows_t<LPR, 1, false>(P, rb, ctas, smem, st);
        case 2: return launch_rows_t<LPR, 2, false>(P, rb, ctas, smem, st);
        default: return launch_rows_t<LPR, 3, false>(P, rb, ctas, smem, st);
    }
}

int sm_count() {
    static int count[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (count[dev] == 0) {
        int c = 0;
        if (cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || c <= 0) c = 148;
        count[dev] = c;
    }
    return count[dev];
}

// Fewest rows whose bf16 scales (G per row) fill whole 16-byte units: 8, 4, 2 or 1.
uint32_t rows_unit(uint32_t G) {
    uint32_t u = 8;
    while (u > 1 && (u / 2u) * G % 8u == 0) u /= 2u;
    return u;
}

// Rows per CTA: an even split of all rows over two CTAs per SM, rounded up to a
// multiple of rows_unit(G) so that ranges of scale rows start on 16-byte boundaries.
uint32_t rows_per_cta(uint32_t total_rows, uint32_t G) {
    const uint32_t ctas = 2u * (uint32_t)sm_count(), u = rows_unit(G);
    const uint32_t rb = (total_rows + ctas - 1) / ctas;
    return (rb + u - 1) / u * u;
}

// One token, 4-bit affine rows of whole 16-byte units, groups of whole units,
// at most 96 units (k <= 3072) per row, and the CTA's shared memory within budget.
bool rows_ok(const QmmArgs &a) {
    if (a.m != 1 || a.n_expert_used > ROWS_MAX_PAIRS || !dp4a_ok(a)) return false;
    const uint32_t xsz = a.x_dtype == DT_F32 ? 4u : 2u;
    if ((a.k * xsz) % 16u != 0 || (uintptr_t)a.x % 16u != 0) return false;
    int lpr, upl;
    rows_shape(a.row_bytes / 16u, &lpr, &upl);
    if (lpr == 0) return false;
    const uint64_t total = (uint64_t)a.n_expert_used * a.out_n;  // rows of the walk
    if (total >= (1ull << 31)) return false;
    const uint32_t rb = rows_per_cta((uint32_t)total, a.groups);
    const uint32_t areas = a.act >= 0 ? 2u : 1u;
    const RowsLayout L = rows_layout(areas * rb, a.row_bytes, a.k * xsz, a.row_bytes / 16u, a.groups);
    return L.total <= 110u * 1024u;
}

cudaError_t launch_rows(GemvParams P, const QmmArgs &a, cudaStream_t st) {
    int lpr, upl;
    rows_shape(P.n_units, &lpr, &upl);
    const uint32_t total = P.R * P.out_n;  // rows of the walk: output elements of a pair
    const uint32_t rb = rows_per_cta(total, P.groups);
    const uint32_t ctas = (total + rb - 1) / rb;
    const uint32_t xsz = a.x_dtype == DT_F32 ? 4u : 2u;
    const uint32_t areas = P.glu_nh ? 2u : 1u;
    const RowsLayout L = rows_layout(areas * rb, P.row_bytes, a.k * xsz, P.n_units, P.groups);
    // with out_n a multiple of u = rows_unit(G), every range a CTA copies (gate and up
    // halves alike) starts and ends on a multiple of u rows, whose scales fill whole
    // 16-byte units
    P.s_bulk = (a.out_n % rows_unit(P.groups)) == 0 && (uintptr_t)a.scales % 16u == 0 &&
               (uintptr_t)a.aux % 16u == 0;
    switch (lpr) {
        case 4: return launch_rows_l<4>(P, upl, rb, ctas, L.total, st);
        case 8: return launch_rows_l<8>(P, upl, rb, ctas, L.total, st);
        case 16: return launch_rows_l<16>(P, upl, rb, ctas, L.total, st);
        default: return launch_rows_l<32>(P, upl, rb, ctas, L.total, st);
    }
}

int tma_lpr(uint32_t nu) {
    // lanes per row: about 3 to 6 16-byte units per lane
    if (nu <= 24) return 4;
    if (nu <= 48) return 8;
    if (nu <= 96) return 16;
    return 32;
}

template <int NPB, int MODE, int LPR>
cudaError_t launch_tma_one(const GemvParams &P, uint32_t ycount, cudaStream_t st) {
    constexpr uint32_t RB = TMA_THREADS / LPR;
    const uint32_t xsz = P.x_dtype == DT_F32 ? 4u : 2u;
    const bool spec = MODE != MODE_ROUTED && P.x_spec;
    const TmaLayout L = tma_layout(RB, P.row_bytes, spec ? P.m * P.k * xsz : NPB * P.k * xsz, NPB,
                                   P.n_units, P.groups);
    auto kern = gemv_aff4_tma<NPB, MODE, LPR>;
    if (L.total > 48 * 1024) {
        static int smem_set[64];
        cudaError_t e = ensure_dyn_smem(kern, L.total, smem_set);
        if (e != cudaSuccess) return e;
    }
    dim3 grid((P.n + RB - 1) / RB, ycount);
    kern<<<grid, TMA_THREADS, L.total, st>>>(P);
    return cudaGetLastError();
}

template <int MODE, int LPR>
cudaError_t launch_tma_npb(const GemvParams &P, uint32_t npb, uint32_t ycount, cudaStream_t st) {
    if (npb <= 1) return launch_tma_one<1, MODE, LPR>(P, ycount, st);
    if (npb <= 2) return launch_tma_one<2, MODE, LPR>(P, ycount, st);
    if (npb <= 4) return launch_tma_one<4, MODE, LPR>(P, ycount, st);
    return launch_tma_one<8, MODE, LPR>(P, ycount, st);
}

template <int MODE>
cudaError_t launch_tma(const GemvParams &P, uint32_t npb, uint32_t ycount, cudaStream_t st) {
    switch (tma_lpr(P.n_units)) {
        case 4: return launch_tma_npb<MODE, 4>(P, npb, ycount, st);
        case 8: return launch_tma_npb<MODE, 8>(P, npb, ycount, st);
        case 16: return launch_tma_npb<MODE, 16>(P, npb, ycount, st);
        default: return launch_tma_npb<MODE, 32>(P, npb, ycount, st);
    }
}

// The TMA kernel needs the DP4A conditions, 16-byte aligned x rows, and its
// shared-memory layout within budget for the largest pair batch.
bool tma_ok(const QmmArgs &a, uint32_t npb, bool spec) {
    if (!dp4a_ok(a)) return false;
    const uint32_t xsz = a.x_dtype == DT_F32 ? 4u : 2u;
    if ((a.k * xsz) % 16u != 0 || (uintptr_t)a.x % 16u != 0) return false;
    const uint32_t nu = a.row_bytes / 16u;
    const uint32_t rb = TMA_THREADS / (uint32_t)tma_lpr(nu);
    const TmaLayout L = tma_layout(rb, a.row_bytes, spec ? a.m * a.k * xsz : npb * a.k * xsz, npb, nu,
                                   a.groups);
    return L.total <= 100u * 1024u;
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
        case K_MXFP4: return launch_npb<K_MXFP4, FUSED>(P, npb, grid, st);
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
        case K_MXFP4: return UnitShape<K_MXFP4>::UC;
        default: return UnitShape<K_NVFP4>::UC;
    }
}

int unit_bytes(int kind) { return kind == K_AFF6 ? 48 : 16; }

GemvParams make_params(const QmmArgs &a, uint32_t *err) {
    GemvParams P{};
    P.x = a.x; P.ids = a.ids; P.packed = a.packed; P.scales = a.scales; P.aux = a.aux;
    P.out = a.out; P.err = err;
    P.R = a.m * a.n_expert_used;
    P.m = a.m;
    P.k = a.k; P.n = a.n; P.gs = a.group_size; P.groups = a.groups;
    P.n_expert_used = a.n_expert_used; P.num_experts = a.num_experts; P.row_bytes = a.row_bytes;
    const uint32_t uc = (uint32_t)unit_codes(a.kind), ub = (uint32_t)unit_bytes(a.kind);
    // units covering the row's bytes (and so all k codes)
    P.n_units = (a.row_bytes + ub - 1) / ub;
    if ((uint64_t)P.n_units * uc < a.k) P.n_units = (a.k + uc - 1) / uc;
    P.xstride = P.n_units * (uc + 1);
    P.x_dtype = a.x_dtype; P.out_dtype = a.out_dtype;
    P.bias = a.bias; P.bias_dtype = a.bias_dtype;
    P.glu_nh = a.act >= 0 ? a.n / 2u : 0u;
    P.out_n = a.out_n;
    P.act = a.act;
    P.pdl = (a.launch_flags & MOE_LAUNCH_PDL) != 0;
    P.early_weights = (a.launch_flags & MOE_LAUNCH_EARLY_WEIGHTS) != 0;
    P.packed_ptrs = a.packed_ptrs; P.scale_ptrs = a.scale_ptrs; P.bias_ptrs = a.bias_ptrs;
    P.fault_ns = a.fault_wait_ns;
    const bool al16 = ((uintptr_t)a.packed % 16 == 0) && (a.row_bytes % 16 == 0);
    const bool al4 = ((uintptr_t)a.packed % 4 == 0) && (a.row_bytes % 4 == 0);
    P.load_mode = al16 ? 16 : al4 ? 4 : 1;
    return P;
}

// Pairs per pass of a decode CTA over its expert's rows: the smallest power of two
// at or above the mean pairs per expert, ceil(R / num_experts), at most min(m, 8).
// Every pass computes NPB pair slots, so a batch much larger than an expert's
// pairs computes mostly empty slots; experts with more pairs take several passes.
uint32_t pairs_per_pass(const QmmArgs &a) {
    const uint64_t R = (uint64_t)a.m * a.n_expert_used;
    const uint64_t mean = (R + a.num_experts - 1) / a.num_experts;
    uint32_t npb = 1;
    while (npb < mean && npb < 8u) npb <<= 1;
    return tmin<uint32_t>(npb, tmin<uint32_t>(a.m, 8u));
}

}  // namespace

cudaError_t launch_gemv_fused(const QmmArgs &a, uint32_t *err, cudaStream_t st) {
    GemvParams P = make_params(a, err);
    const uint32_t distinct_max = min(P.R, a.num_experts);
    dim3 grid((a.n + GEMV_ROWS - 1) / GEMV_ROWS, distinct_max);
    // pairs of one expert come from distinct tokens unless ids repeat inside a token
    const uint32_t npb = pairs_per_pass(a);
    const uint32_t xsz = a.x_dtype == DT_F32 ? 4u : 2u;
    const bool spec = (uint64_t)a.m * a.k * xsz <= 32768u;
    if (a.packed_ptrs) return launch_kind<true>(P, a.kind, npb, grid, st);  // pointer-table weights
    if (rows_ok(a)) return launch_rows(P, a, st);
    if (a.act >= 0) return launch_kind<true>(P, a.kind, npb, grid, st);  // gated output
    if (a.m == 1 && tma_ok(a, 1, spec)) {
        P.x_spec = spec;
        return launch_tma<MODE_PAIR>(P, 1, P.R, st);
    }
    if (tma_ok(a, npb, spec)) {
        P.x_spec = spec;
        return launch_tma<MODE_FUSED>(P, npb, distinct_max, st);
    }
    if (dp4a_ok(a)) return launch_dp4a<true>(P, npb, grid, st);
    return launch_kind<true>(P, a.kind, npb, grid, st);
}

cudaError_t launch_gemv_routed(const QmmArgs &a, const uint32_t *counts, const uint32_t *offsets,
                               const uint32_t *sorted_pairs, uint32_t *err, cudaStream_t st) {
    GemvParams P = make_params(a, err);
    P.counts = counts; P.offsets = offsets; P.sorted_pairs = sorted_pairs;
    dim3 grid((a.n + GEMV_ROWS - 1) / GEMV_ROWS, a.num_experts);
    const uint32_t npb = pairs_per_pass(a);
    if (a.packed_ptrs || a.act >= 0) return launch_kind<false>(P, a.kind, npb, grid, st);  // pointer tables, gated output
    if (tma_ok(a, npb, false)) return launch_tma<MODE_ROUTED>(P, npb, a.num_experts, st);
    if (dp4a_ok(a)) return launch_dp4a<false>(P, npb, grid, st);
    return launch_kind<false>(P, a.kind, npb, grid, st);
}

}  // namespace moe
