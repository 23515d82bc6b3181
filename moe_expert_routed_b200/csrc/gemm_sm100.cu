// gemm_sm100.cu -- expert-grouped GEMM on the 5th-generation tensor cores (tcgen05).
//
// A persistent grid (one CTA per SM) walks work items: a 128 x BN tile of one
// expert, 128 consecutive weight rows (output columns) of expert e against up to
// BN of the (token, slot) pairs routed to e (a tile of the routing prologue's
// tile list). Operands are
// swapped relative to out = x * W^T: the dequantised weight tile is the MMA's
// A operand (M = 128) and the gathered token rows are B (N = pairs in the tile,
// rounded up to 16), so each weight tile is dequantised once per tile of pairs.
// The pages' designs that this replaces: fused Metal dequant to fp16 followed
// by gather_mm (turboquant fast_switch_patch.py) and the routed W4A16 grouped
// GEMM fed by expert_offsets / sorted_token_ids (metrale helpers_b.rs,
// launch_grouped_gemm).
//
// Warp roles (736 threads), each running through the CTA's items and their
// k-tiles on its own; the stage ring continues from one item to the next:
//   warps 0-7   dequantisers: per 64-wide k-tile, turn the staged codes of 128
//               rows x 64 codes into 16-bit values: into tensor memory
//               (tcgen05.st, one lane quarter per warp) for the two-term formats
//               with tiles of up to 128 pairs, else into shared memory in the
//               128-byte-swizzled K-major layout (and split f32 x into two bf16
//               halves when the loaders copied it).
//   warps 8-15  loaders: cp.async the pairs' x rows straight into the B operand
//               tile and the packed codes and scale words into a staging area,
//               up to S k-tiles ahead of the tensor core; each loader's
//               completion is signalled on the stage's mbarrier by the copy
//               engine (cp.async.mbarrier.arrive), so loaders never block on
//               their own copies.
//   warp 16     TMEM allocation; one lane issues tcgen05.mma (kind::f16, fp32
//               accumulation in TMEM; A from tensor or shared memory, B from
//               shared memory) and tcgen05.commit.
//   warp 17     with TMA staging, one lane issues the k-tiles' tensor copies of
//               the packed codes (no multicast), S k-tiles ahead like the loaders.
//   warps 18-21 epilogue: TMEM -> registers (tcgen05.ld), times scale2 for
//               NVFP4, rounded once to the output type, stored to row p of out
//               (the scatter back to [token][slot] order). Two TMEM accumulators
//               alternate between items, so an item's epilogue overlaps the next
//               item's MMAs.
//   warp 22     scheduler: one lane claims work items (each CTA's first is its
//               block index, the rest come from an atomic counter, so that CTAs
//               that finish early take more) and publishes them to the other
//               roles through a 4-slot ring in shared memory.
// Per stage: loaded (loader copies landed) -> full (dequantised) -> empty (the
// MMAs that read it completed). Dequantisation of k-tile kt overlaps the MMAs
// of kt-1 and the copies of kt+1 .. kt+S-1. Every wait is bounded (1 s); a wait
// that gives up sets ERR_TIMEOUT, the CTA drains its in-flight MMAs and copies,
// frees TMEM and exits.
//
// Exactness: products must stay exact so that the fp32 accumulation is the
// only rounding. NVFP4 weights e2m1 * e4m3 have at most 6 significant bits and
// are exact in bf16/f16: one MMA per k-step. Affine (c*s + b) and codebook
// (cb[c]*s) weights are formed in fp32 and split into a 16-bit high part and
// the 16-bit rounding of the remainder (two MMAs). f32 x is split the same way
// into two bf16 halves; the lo*lo product is dropped (below 2^-16 relative).
#include <string.h>

#include <cuda.h>  // CUtensorMap and its encoding enums (the driver is reached via cudaGetDriverEntryPoint)
#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace moe {

namespace {

constexpr int BM = 128;
constexpr int KT = 64;                          // k per tile: one 128-byte swizzle atom of 16-bit values
constexpr int NDQ = 256;                        // dequantising threads (warps 0-7)
constexpr int NLD = 256;                        // loader threads (warps 8-15)
constexpr int NEP = 128;                        // epilogue threads (warps 18-21)
constexpr int GEMM_THREADS = NDQ + NLD + 64 + NEP + 32;  // + the MMA, tensor-copy and scheduler warps
constexpr int LD_WARP0 = NDQ / 32;
constexpr int MMA_WARP = (NDQ + NLD) / 32;
constexpr int TMA_WARP = MMA_WARP + 1;
constexpr int EPI_WARP0 = TMA_WARP + 1;
constexpr int SCHED_WARP = EPI_WARP0 + NEP / 32;
// how the B operand's x rows reach shared memory
constexpr uint32_t XM_LOADERS = 0;  // 16-byte copies by the loader warps
constexpr uint32_t XM_ROWS = 1;     // tensor copies of x rows gathered into expert order beforehand
constexpr uint32_t XM_IMAGE = 2;    // one bulk copy per k-tile of the tile-major, pre-swizzled f16 image
constexpr uint32_t RING = 4;                    // work items the scheduler may publish ahead
// arrivals that release a ring slot: one per dequantiser, loader and epilogue warp,
// plus the tensor-copy and MMA lanes
constexpr uint32_t RING_READERS = NDQ / 32 + NLD / 32 + NEP / 32 + 2;
constexpr int MAX_STAGES = 6;
constexpr int A_TILE = BM * KT * 2;             // bytes per A term per stage
constexpr uint64_t WAIT_NS = 1000000000ull;
// limit of the waits that let a CTA's own copies and MMAs complete after another
// wait gave up (independent of the pipeline waits' limit)
constexpr uint64_t DRAIN_NS = 1000000000ull;

struct GemmParams {
    const void *x;
    const uint32_t *offsets, *sorted_pairs, *tiles, *tile_count;
    const uint8_t *packed;
    const void *scales;
    const void *aux;
    void *out;
    uint32_t *err;
    uint32_t k, n, lg_gs, groups, n_expert_used, row_bytes, ktiles, stages;
    uint32_t scale_words;  // rows of scales (and biases) 4-byte aligned: staged by the loaders
    uint32_t raw16;        // rows of codes 16-byte aligned: staged in 16-byte copies (else 8)
    const void *bias;      // per-expert output bias [num_experts, n] (bias_dtype), or null
    int bias_dtype;
    // pointer-table weights (null: contiguous arrays): per-expert base addresses of
    // the packed rows, scales and affine biases; a null packed entry skips the expert
    const uint64_t *packed_ptrs, *scale_ptrs, *bias_ptrs;
    int out_dtype;
    uint64_t timeout_ns;
    // gated output (0: plain): tile rows alternate gate and up weight rows (glu_row),
    // and the epilogue writes act(gate) * up into rows of glu_nh = n/2 columns
    uint32_t glu_nh;
    int act;
    uint32_t n_mtiles;      // 128-row blocks per expert (work items per tile)
    // x tiles (XM_*): XM_ROWS reads the x rows gathered in expert order (f32 x: bf16 high
    // halves in rows [0, xg_R), remainders in rows [xg_R, 2 xg_R)) through the kernel's
    // second tensor map
    uint32_t xmode;
    uint32_t xg_R;
    // W4A4, or the f16 image of bf16 x: per-token factor of every output (null: none)
    const float *tok_scale;
    // XM_IMAGE: the B operand image, tile t's k-tile kt at (t * ktiles + kt) * BN * 128
    const uint8_t *ximage;
    uint32_t *work_counter; // items claimed beyond each CTA's first (zeroed by the routing prologue)
    // failure-detection test hook: non-zero makes the MMA warp first wait this long on
    // a barrier nothing completes (so the CTA aborts); 0 in normal operation
    uint64_t fault_ns;
    // packed codes staged by TMA tensor copies (the kernel's tensor-map argument) instead
    // of the loaders' cp.async
    uint32_t tma;
};

// 16-bit terms of the A operand: NVFP4 e2m1 * e4m3 and MXFP4 e2m1 * 2^e are exact in
// one bf16 (or f16) value; affine and codebook weights take a hi and a lo term.
template <int KIND> constexpr int a_terms() { return (KIND == K_NVFP4 || KIND == K_MXFP4) ? 1 : 2; }

// Byte offset of 16-byte chunk c (0..7) of row r inside a swizzled K-major tile.
__device__ __forceinline__ uint32_t swz(uint32_t r, uint32_t c) {
    return (r >> 3) * 1024u + (r & 7u) * 128u + ((c ^ (r & 7u)) << 4);
}

__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
                 "r"(d)
                 : "memory");
}

template <bool F16>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
    if constexpr (F16) {
        __half2 h = __floats2half2_rn(lo, hi);
        return *reinterpret_cast<uint32_t *>(&h);
    } else {
        __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
        return *reinterpret_cast<uint32_t *>(&h);
    }
}

// The two values of a packed 16-bit pair back as floats (exact).
template <bool F16>
__device__ __forceinline__ float2 unpack2(uint32_t p) {
    if constexpr (F16) {
        return __half22float2(*reinterpret_cast<const __half2 *>(&p));
    } else {
        return make_float2(__uint_as_float(p << 16), __uint_as_float(p & 0xFFFF0000u));
    }
}

// Packed words holding one thread's 32 codes (j0 a multiple of 32).
template <int KIND> struct Raw;
template <> struct Raw<K_AFF4> { static constexpr int W = 4; };
template <> struct Raw<K_CB4> { static constexpr int W = 4; };
template <> struct Raw<K_NVFP4> { static constexpr int W = 4; };
template <> struct Raw<K_MXFP4> { static constexpr int W = 4; };
template <> struct Raw<K_AFF8> { static constexpr int W = 8; };
template <> struct Raw<K_AFF6> { static constexpr int W = 6; };
template <> struct Raw<K_CB2> { static constexpr int W = 2; };
template <> struct Raw<K_CB3> { static constexpr int W = 4; };  // codes SUB .. SUB+31, SUB <= 8

// Staging area of one k-tile: one row per weight row,
//   bytes [0, RB)         the k-tile's packed codes (3-bit codebook: the 8 words
//                         from word floor(j0/10), which hold codes j0 .. j0+63)
//   bytes [RB, RB+8)      the 4-byte-aligned scale word(s) holding the k-tile's groups
//   bytes [RB+8, RB+16)   the same words of the biases (affine)
// Rows are an odd number of 16-byte units apart, so 8 consecutive rows read
// with 16-byte loads touch all 32 banks once.
//
// With TMA staging (contiguous weights, rows a multiple of 16 bytes) the same area
// holds instead
//   [0, BM*RB)            the codes, BM rows of RB bytes written by two 64-row
//                         tensor copies; for RB = 32 / 64 the 16-byte chunks of a
//                         row are swizzled within 32 / 64 bytes (the copies'
//                         SWIZZLE_32B / 64B mode), so 8 consecutive rows read with
//                         16-byte loads touch all 32 banks once
//   [BM*RB, BM*RB+BM*16)  per row: scale words (8 bytes), then bias words (8 bytes)
// 3-bit codebook rows (10 codes per word) are a multiple of 8 bytes, so two rows
// form a "super-row" of a multiple of 16 bytes and the codes come as two tensor
// copies of 64 super-rows x CB3_WIN bytes: the window of the k-tile's words in the
// even rows, then in the odd rows, each starting at the 16-byte boundary below
// the k-tile's first word:
//   [0, 64*CB3_WIN)              even rows 0, 2, ..., 126
//   [64*CB3_WIN, 128*CB3_WIN)    odd rows 1, 3, ..., 127
//   [128*CB3_WIN, +BM*16)        scale and bias words as above
constexpr uint32_t CB3_WIN = 48;  // up to 12 bytes of offset + 8 words of 10 codes
template <int KIND> struct RawLayout {
    static constexpr uint32_t RB = KIND == K_CB3 ? 32u : 8u * kind_bits(KIND);
    static constexpr uint32_t SC = RB;  // scale words at SC, bias words at SC + 8
    static constexpr uint32_t STRIDE = ((RB + 16u) / 16u) % 2u ? RB + 16u : RB + 32u;
    static constexpr uint32_t TMA_SC = KIND == K_CB3 ? BM * CB3_WIN : BM * RB;
    static constexpr uint32_t TILE = KIND == K_CB3 ? BM * CB3_WIN + BM * 16u : BM * STRIDE;
    static_assert(TMA_SC + BM * 16u <= TILE && BM * STRIDE <= TILE, "both stagings fit the area");
};

// Byte offset of 16-byte chunk c of staged row sr in the TMA code tile (the
// swizzle the tensor copies apply: address bit 4 ^= bit 7 for 32-byte rows, bits
// 4-5 ^= bits 7-8 for 64-byte rows; the tile is 1024-byte aligned).
template <int KIND>
__device__ __forceinline__ uint32_t tma_chunk(uint32_t sr, uint32_t c) {
    constexpr uint32_t RB = RawLayout<KIND>::RB;
    if constexpr (RB == 32) return sr * 32u + 16u * (c ^ ((sr >> 2) & 1u));
    else if constexpr (RB == 64) return sr * 64u + 16u * (c ^ ((sr >> 1) & 3u));
    else return sr * RB + 16u * c;
}

template <int KIND, int SUB>
__device__ __forceinline__ uint32_t raw_code(const uint32_t (&w)[Raw<KIND>::W], int i) {
    // i is a compile-time constant after unrolling
    if constexpr (KIND == K_AFF4 || KIND == K_CB4 || KIND == K_NVFP4 || KIND == K_MXFP4) {
        return (w[i / 8] >> (4 * (i % 8))) & 15u;
    } else if constexpr (KIND == K_AFF8) {
        return (w[i / 4] >> (8 * (i % 4))) & 255u;
    } else if constexpr (KIND == K_CB2) {
        return (w[i / 16] >> (2 * (i % 16))) & 3u;
    } else if constexpr (KIND == K_AFF6) {
        const int b = 6 * i, wi = b / 32, sh = b % 32;
        return sh <= 26 ? (w[wi] >> sh) & 63u : __funnelshift_r(w[wi], w[wi + 1 < 6 ? wi + 1 : wi], sh) & 63u;
    } else {  // K_CB3: code (SUB + i) of the loaded words, 10 codes per word
        return (w[(SUB + i) / 10] >> (3 * ((SUB + i) % 10))) & 7u;
    }
}

template <int KIND, int SUB>
__device__ __forceinline__ void dequant32(const uint32_t (&w)[Raw<KIND>::W], float s0, float b0,
                                          float s1, float b1, bool two_groups, const float *cb,
                                          float (&v)[32]) {
#pragma unroll
    for (int i = 0; i < 32; i++) {
        const uint32_t code = raw_code<KIND, SUB>(w, i);
        const float s = (i >= 16 && two_groups) ? s1 : s0;
        const float b = (i >= 16 && two_groups) ? b1 : b0;
        if constexpr (KIND == K_AFF4 || KIND == K_AFF6 || KIND == K_AFF8) v[i] = fmaf((float)code, s, b);
        else if constexpr (KIND == K_MXFP4) v[i] = e2m1_to_f32(code) * s;  // s = 2^(e - 127): exact
        else v[i] = cb[code] * s;
    }
}

// Store 32 fp32 weights as 4 chunks of 8 16-bit values at chunk positions
// c0..c0+3 of row r: the 16-bit rounding (hi) and, for two-term formats, the
// 16-bit rounding of the remainder (lo). TM: into the words hw / lw instead (word
// j holds values 2j and 2j+1), for a store to tensor memory.
template <bool F16, bool TWO, bool TM = false>
__device__ __forceinline__ void store_a(const float (&v)[32], uint32_t a_hi, uint32_t a_lo, uint32_t r,
                                        uint32_t c0, uint32_t (&hw)[16], uint32_t (&lw)[16]) {
#pragma unroll
    for (int cc = 0; cc < 4; cc++) {
        uint32_t hh[4], ll[4];
#pragma unroll
        for (int e = 0; e < 4; e++) {
            const float x0 = v[cc * 8 + 2 * e], x1 = v[cc * 8 + 2 * e + 1];
            hh[e] = pack2<F16>(x0, x1);
            if constexpr (TWO) {
                const float2 h = unpack2<F16>(hh[e]);
                ll[e] = pack2<F16>(x0 - h.x, x1 - h.y);
            }
        }
        if constexpr (TM) {
#pragma unroll
            for (int e = 0; e < 4; e++) {
                hw[cc * 4 + e] = hh[e];
                if constexpr (TWO) lw[cc * 4 + e] = ll[e];
            }
        } else {
            const uint32_t off = swz(r, c0 + cc);
            sts128(a_hi + off, hh[0], hh[1], hh[2], hh[3]);
            if constexpr (TWO) sts128(a_lo + off, ll[0], ll[1], ll[2], ll[3]);
        }
    }
}

// Two E4M3 bytes (low byte first) to f16x2 by the hardware conversion.
__device__ __forceinline__ __half2 e4m3x2_to_half2(uint32_t two) {
    uint32_t h;
    asm("{\n\t.reg .b16 t;\n\tcvt.u16.u32 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}" : "=r"(h) : "r"(two));
    return *reinterpret_cast<__half2 *>(&h);
}

// NVFP4: e2m1 pairs to f16x2 by the hardware conversion, times the E4M3 block
// scales s01 = (s0, s1) as an f16 multiply (exact: at most 6 significant bits,
// magnitudes in [2^-10, 2688]), stored as f16, or as bf16 through f32 (exact).
// Codes 0-15 of the thread's 32 belong to the group of s0, codes 16-31 to s1.
template <bool F16>
__device__ __forceinline__ void nvfp4_store(const uint32_t (&w)[4], __half2 s01, uint32_t a_hi, uint32_t r,
                                            uint32_t c0) {
    const __half2 sa = __low2half2(s01), sb = __high2half2(s01);
#pragma unroll
    for (int cc = 0; cc < 4; cc++) {  // word cc holds codes 8cc .. 8cc+7
        uint32_t h[4];
        asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
            "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
            "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
            "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
            "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
            "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
            : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
            : "r"(w[cc]));
        const __half2 sc = cc >= 2 ? sb : sa;
        uint32_t o[4];
#pragma unroll
        for (int e = 0; e < 4; e++) {
            const __half2 pr = __hmul2(*reinterpret_cast<const __half2 *>(&h[e]), sc);
            if constexpr (F16) {
                o[e] = *reinterpret_cast<const uint32_t *>(&pr);
            } else {
                const float2 f = __half22float2(pr);
                o[e] = pack2<false>(f.x, f.y);
            }
        }
        sts128(a_hi + swz(r, c0 + cc), o[0], o[1], o[2], o[3]);
    }
}

// Codebook weights with f16 x (A in f16): each code pair (2e, 2e+1) of the thread's
// 32 codes is looked up as one f16x2 (cb[c0], cb[c1]) in a pair table of
// 2^(2 bits) entries, then w = cb * s is split into hi = f16(cb * s) and
// lo = f16(cb * s - hi) by an f16x2 multiply and a fused multiply-add. cb and s
// are f16, so cb * s has at most 22 significant bits and hi + lo holds it to
// within the f16 subnormal spacing (2^-24). Codes of a pair share a word (pairs
// start at even positions and a 3-bit word holds 10 codes).
template <int KIND, int SUB, bool TM = false>
__device__ __forceinline__ void cb_pairs_f16(const uint32_t (&w)[Raw<KIND>::W], __half2 s0, __half2 s1,
                                             bool two_groups, const uint32_t *lut2, uint32_t a_hi,
                                             uint32_t a_lo, uint32_t r, uint32_t c0, uint32_t (&hw)[16],
                                             uint32_t (&lw)[16]) {
    constexpr int B = kind_bits(KIND);
#pragma unroll
    for (int cc = 0; cc < 4; cc++) {
        uint32_t hh[4], ll[4];
#pragma unroll
        for (int e = 0; e < 4; e++) {
            const int i = cc * 8 + 2 * e;  // first code of the pair (compile-time)
            uint32_t idx;
            if constexpr (KIND == K_CB3) {
                idx = (w[(SUB + i) / 10] >> (3 * ((SUB + i) % 10))) & 63u;
            } else {
                constexpr int EPW = 32 / B;
                idx = (w[i / EPW] >> (B * (i % EPW))) & ((1u << (2 * B)) - 1u);
            }
            const uint32_t pr = lut2[idx];
            const __half2 cbp = *reinterpret_cast<const __half2 *>(&pr);
            const __half2 sv = (i >= 16 && two_groups) ? s1 : s0;
            const __half2 hi = __hmul2(cbp, sv);
            const __half2 lo = __hfma2(cbp, sv, __hneg2(hi));
            hh[e] = *reinterpret_cast<const uint32_t *>(&hi);
            ll[e] = *reinterpret_cast<const uint32_t *>(&lo);
        }
        if constexpr (TM) {
#pragma unroll
            for (int e = 0; e < 4; e++) {
                hw[cc * 4 + e] = hh[e];
                lw[cc * 4 + e] = ll[e];
            }
        } else {
            const uint32_t off = swz(r, c0 + cc);
            sts128(a_hi + off, hh[0], hh[1], hh[2], hh[3]);
            sts128(a_lo + off, ll[0], ll[1], ll[2], ll[3]);
        }
    }
}

template <int KIND, bool F16, bool TM = false>
__device__ __forceinline__ void dequant_tile(const uint32_t (&w)[Raw<KIND>::W], uint32_t sub, float s0,
                                             float b0, float s1, float b1, bool two_groups,
                                             const float *cb, uint32_t a_hi, uint32_t a_lo, uint32_t r,
                                             uint32_t c0, uint32_t (&hw)[16], uint32_t (&lw)[16]) {
    static_assert(KIND != K_NVFP4, "NVFP4 tiles go through nvfp4_store");
    constexpr bool TWO = a_terms<KIND>() == 2;
    {
        float v[32];
        if constexpr (KIND == K_CB3) {
            switch (sub) {  // first code's position in word 0: 0, 2, 4, 6 or 8
                case 0: dequant32<KIND, 0>(w, s0, b0, s1, b1, two_groups, cb, v); break;
                case 2: dequant32<KIND, 2>(w, s0, b0, s1, b1, two_groups, cb, v); break;
                case 4: dequant32<KIND, 4>(w, s0, b0, s1, b1, two_groups, cb, v); break;
                case 6: dequant32<KIND, 6>(w, s0, b0, s1, b1, two_groups, cb, v); break;
                default: dequant32<KIND, 8>(w, s0, b0, s1, b1, two_groups, cb, v); break;
            }
        } else {
            dequant32<KIND, 0>(w, s0, b0, s1, b1, two_groups, cb, v);
        }
        store_a<F16, TWO, TM>(v, a_hi, a_lo, r, c0, hw, lw);
    }
}

// Scale (and bias) whose first byte lies `rel` bytes after the start of the
// staged scale words sw / bias words bw.
template <int KIND>
__device__ __forceinline__ void staged_scale(const uint32_t (&sw)[2], const uint32_t (&bw)[2], uint32_t rel,
                                             float &s, float &b) {
    const uint32_t wi = rel >> 2, sh = (rel & 3u) * 8u;
    const uint32_t sv = (wi ? sw[1] : sw[0]) >> sh;
    if constexpr (KIND == K_NVFP4) {
        s = e4m3_to_f32(sv & 0xFFu);
        b = 0.f;
    } else if constexpr (KIND == K_MXFP4) {
        s = e8m0_to_f32(sv & 0xFFu);
        b = 0.f;
    } else if constexpr (KIND == K_AFF4 || KIND == K_AFF6 || KIND == K_AFF8) {
        s = bf16_bits_to_f32(sv & 0xFFFFu);
        b = bf16_bits_to_f32(((wi ? bw[1] : bw[0]) >> sh) & 0xFFFFu);
    } else {
        s = f16_bits_to_f32(sv & 0xFFFFu);
        b = 0.f;
    }
}

// Scale (and bias) of group g read from global memory (rows of scales that are
// not 4-byte aligned); groups past the row's end read as 0.
template <int KIND>
__device__ __forceinline__ void global_scale(const uint8_t *srow, const uint8_t *brow, uint32_t g,
                                             uint32_t groups, float &s, float &b) {
    s = 0.f;
    b = 0.f;
    if (g >= groups) return;
    if constexpr (KIND == K_NVFP4) {
        s = e4m3_to_f32(__ldg(srow + g));
    } else if constexpr (KIND == K_MXFP4) {
        s = e8m0_to_f32(__ldg(srow + g));
    } else {
        const uint32_t sv = (uint32_t)__ldg(srow + 2 * g) | ((uint32_t)__ldg(srow + 2 * g + 1) << 8);
        if constexpr (KIND == K_AFF4 || KIND == K_AFF6 || KIND == K_AFF8) {
            s = bf16_bits_to_f32(sv);
            b = bf16_bits_to_f32((uint32_t)__ldg(brow + 2 * g) | ((uint32_t)__ldg(brow + 2 * g + 1) << 8));
        } else {
            s = f16_bits_to_f32(sv);
        }
    }
}

// ATM: the two-term A operand (affine, codebook) of tiles up to 128 pairs wide lives
// in tensor memory: the dequantisers store it with tcgen05.st and the MMAs read it
// from there (A_TM_COLS columns per term and stage after the two accumulators), so
// the stage in shared memory holds only B and the staged codes. Wider tiles leave no
// room beside their accumulators and keep A in shared memory.
constexpr uint32_t A_TM_COLS = KT / 2;  // 16-bit values, two per 32-bit column
template <int KIND, int XT, int BN>
struct GemmCfg {
    static constexpr int AT = a_terms<KIND>();
    static constexpr int BT = (XT == DT_F32) ? 2 : 1;
    static constexpr bool ATM = AT == 2 && BN <= 128;
    static constexpr int B_TILE = BN * KT * 2;
    static constexpr uint32_t STAGE = (ATM ? 0u : AT * A_TILE) + BT * B_TILE + RawLayout<KIND>::TILE;
};

// Work item w of the persistent grid: tile w / n_mtiles of the routing prologue's
// tile list (expert e, first pair r0 of the expert's pairs) and 128-row block
// w % n_mtiles of the expert's weight rows. Every role of a CTA walks the same
// items (read from the scheduler's ring) and evaluates the same item set-up, so
// they agree on which items are skipped.
template <int KIND, bool PTRS>
struct Item {
    uint32_t e, r0, off, nt, nt_pad, row0;
    const uint8_t *wb, *sb, *bb;
    bool ptr_scale_words, ptr_raw16;

    // false when the item is skipped (pointer-table expert not held here, or with
    // unusable buffers: flagged once per item by block 0 of the column blocks)
    __device__ __forceinline__ bool load(const GemmParams &P, uint32_t t, uint32_t nb, uint32_t bn) {
        constexpr uint32_t ES = (KIND == K_NVFP4 || KIND == K_MXFP4) ? 1u : 2u;
        constexpr bool AFF = (KIND == K_AFF4 || KIND == K_AFF6 || KIND == K_AFF8);
        e = __ldg(P.tiles + 2 * t);
        r0 = __ldg(P.tiles + 2 * t + 1);
        off = __ldg(P.offsets + e);
        const uint32_t cnt = __ldg(P.offsets + e + 1) - off;
        nt = tmin<uint32_t>(bn, cnt - r0);
        nt_pad = (nt + 15u) & ~15u;
        row0 = nb * BM;
        wb = P.packed + (size_t)e * P.n * P.row_bytes;
        sb = (const uint8_t *)P.scales + (size_t)e * P.n * P.groups * ES;
        bb = (const uint8_t *)P.aux + (size_t)e * P.n * P.groups * 2u;
        ptr_scale_words = false;
        ptr_raw16 = false;
        if constexpr (PTRS) {
            wb = (const uint8_t *)__ldg(P.packed_ptrs + e);
            if (!wb) return false;  // expert held elsewhere: its pairs' rows are not ours to write
            sb = (const uint8_t *)__ldg(P.scale_ptrs + e);
            bb = AFF ? (const uint8_t *)__ldg(P.bias_ptrs + e) : nullptr;
            // the copies need 8-byte aligned code rows (4 for 3-bit codebook rows) and 2-byte
            // aligned 16-bit scales / biases; other experts are skipped and flagged
            const uintptr_t wal = KIND == K_CB3 ? 4u : 8u;
            const uintptr_t sal = (uintptr_t)sb | (AFF ? (uintptr_t)bb : 0u);
            if (!sb || (AFF && !bb) || ((uintptr_t)wb % wal) != 0 || (ES == 2u && (sal & 1u))) {
                if (nb == 0 && threadIdx.x == 0) atomicOr(P.err, ERR_BAD_POINTER);
                return false;
            }
            ptr_raw16 = P.raw16 != 0 && (uintptr_t)wb % 16u == 0;
            ptr_scale_words = P.scale_words != 0 && sal % 4u == 0 && (uintptr_t)sb % 4u == 0;
        }
        return true;
    }
};

// Persistent grid, one CTA per SM. PTRS: weights from the pointer tables (decided at
// compile time so that the contiguous case keeps its copy-width and scale-staging
// branches on kernel parameters). GLU: gated output (glu_row order, act(gate) * up
// epilogue), also decided at compile time so that the plain kernels carry none of it.
// XIMG (f16 x only): the B tiles come by one bulk copy per k-tile from the image.
template <int KIND, int XT, int BN, bool PTRS, bool GLU, bool XIMG = false>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
grouped_gemm_kernel(const GemmParams P, const __grid_constant__ CUtensorMap tmap,
                    const __grid_constant__ CUtensorMap xmap) {
    using C = GemmCfg<KIND, XT, BN>;
    static_assert(!XIMG || (XT == DT_F16 && !PTRS && !GLU), "the image is f16, for the plain kernel");
    constexpr int AT = C::AT, BT = C::BT, B_TILE = C::B_TILE;
    constexpr uint32_t STAGE = C::STAGE;
    constexpr bool ATM = C::ATM;
    constexpr uint32_t B_OFF = ATM ? 0u : AT * A_TILE, RAW_OFF = B_OFF + BT * B_TILE;
    constexpr bool F16 = (XT == DT_F16);
    constexpr uint32_t ES = (KIND == K_NVFP4 || KIND == K_MXFP4) ? 1u : 2u;  // bytes per scale
    constexpr bool AFF = (KIND == K_AFF4 || KIND == K_AFF6 || KIND == K_AFF8);
    using RL = RawLayout<KIND>;
    // two TMEM accumulators of BN columns: the epilogue drains one while the MMAs fill
    // the other
    static_assert(BN == 64 || BN == 128 || BN == 256, "tile widths");
    constexpr uint32_t NACC = 2u;
    constexpr uint32_t TMEM_COLS = ATM ? 512u : 2u * BN;
    constexpr uint32_t ACC_STRIDE = BN;
    constexpr uint32_t ACOL0 = 2u * BN;  // ATM: A of stage s, term t at ACOL0 + (s AT + t) A_TM_COLS

    extern __shared__ uint8_t smem_raw[];
    __shared__ uint64_t bars[3 * MAX_STAGES + 6 + 2 * RING];
    __shared__ uint32_t ring_s[RING];
    __shared__ uint32_t tmem_s;
    __shared__ int abort_s;
    __shared__ float cb_s[16];
    // codebook with f16 x: f16x2 table of code pairs (cb[c & mask], cb[c >> bits])
    constexpr bool CBF16 = (KIND == K_CB2 || KIND == K_CB3 || KIND == K_CB4) && XT == DT_F16;
    __shared__ uint32_t lut2_s[CBF16 ? (1u << (2 * kind_bits(KIND))) : 1u];

    const uint32_t tid = threadIdx.x, warp = tid >> 5, lane = tid & 31u;
    const uint32_t S = P.stages;
    const uint32_t nm = P.n_mtiles;  // work items per tile
    const uint32_t n_items = __ldg(P.tile_count) * nm;

    const uint32_t base = (ptx::smem_u32(smem_raw) + 1023u) & ~1023u;
    uint8_t *const base_ptr = smem_raw + (base - ptx::smem_u32(smem_raw));
    const uint32_t full0 = ptx::smem_u32(&bars[0]);
    const uint32_t loaded0 = ptx::smem_u32(&bars[MAX_STAGES]);
    const uint32_t empty0 = ptx::smem_u32(&bars[2 * MAX_STAGES]);
    const uint32_t accfull0 = ptx::smem_u32(&bars[3 * MAX_STAGES]);       // [2]: MMAs of an item done
    const uint32_t accempty0 = ptx::smem_u32(&bars[3 * MAX_STAGES + 2]);  // [2]: epilogue done reading
    const uint32_t drainb = ptx::smem_u32(&bars[3 * MAX_STAGES + 4]);
    const uint32_t never = ptx::smem_u32(&bars[3 * MAX_STAGES + 5]);  // completed by nothing
    const uint32_t ringfull0 = ptx::smem_u32(&bars[3 * MAX_STAGES + 6]);          // [RING]
    const uint32_t ringempty0 = ptx::smem_u32(&bars[3 * MAX_STAGES + 6 + RING]);  // [RING]
    volatile int *abort_flag = &abort_s;
    volatile uint32_t *ring = ring_s;
    // The i-th work item of the CTA from the scheduler's ring (n_items: none left);
    // the slot is released by one arrival per reading warp (lane 0, after the whole
    // warp has read it) or single reading lane. False if the wait gave up.
    auto next_item = [&](uint32_t i, bool whole_warp, uint32_t &w) -> bool {
        const uint32_t slot = i % RING;
        if (!ptx::mbar_wait_bounded(ringfull0 + 8 * slot, (i / RING) & 1u, abort_flag, P.err, ERR_TIMEOUT,
                                    P.timeout_ns))
            return false;
        w = ring[slot];
        if (whole_warp) __syncwarp();
        if (!whole_warp || lane == 0) ptx::mbar_arrive(ringempty0 + 8 * slot);
        return true;
    };

    const bool tma = !PTRS && P.tma != 0;
    // x tiles: by the loader warps' 16-byte copies, or (f32 x) by tensor copies of rows
    // gathered beforehand; a compile-time XM_LOADERS for 16-bit x
    const uint32_t xmode = XIMG ? XM_IMAGE : (XT == DT_F32) ? P.xmode : XM_LOADERS;
    if (tid == 0) {
        for (uint32_t s = 0; s < S; s++) {
            ptx::mbar_init(full0 + 8 * s, NDQ);
            ptx::mbar_init(loaded0 + 8 * s, NLD + ((tma || xmode != XM_LOADERS) ? 1u : 0u));  // + the tensor-copy warp's
            ptx::mbar_init(empty0 + 8 * s, 1);
        }
        for (uint32_t b = 0; b < 2; b++) {
            ptx::mbar_init(accfull0 + 8 * b, 1);
            ptx::mbar_init(accempty0 + 8 * b, NEP / 32);  // one arrival per epilogue warp
        }
        ptx::mbar_init(drainb, 1);
        ptx::mbar_init(never, 1);
        for (uint32_t b = 0; b < RING; b++) {
            ptx::mbar_init(ringfull0 + 8 * b, 1);
            ptx::mbar_init(ringempty0 + 8 * b, RING_READERS);
        }
        ptx::fence_mbar_init();
        abort_s = 0;
    }
    if constexpr (KIND == K_CB2 || KIND == K_CB3 || KIND == K_CB4) {
        if (tid < (1u << kind_bits(KIND)))
            cb_s[tid] = f16_bits_to_f32(__ldg((const unsigned short *)P.aux + tid));
        if constexpr (CBF16) {
            constexpr uint32_t NC = 1u << kind_bits(KIND);
            for (uint32_t i = tid; i < NC * NC; i += blockDim.x) {
                const uint32_t lo = __ldg((const unsigned short *)P.aux + (i & (NC - 1u)));
                const uint32_t hi = __ldg((const unsigned short *)P.aux + (i / NC));
                lut2_s[i] = lo | (hi << 16);
            }
        }
    }
    if (warp == MMA_WARP) {
        ptx::tmem_alloc(ptx::smem_u32(&tmem_s), TMEM_COLS);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = tmem_s;
    const bool gs16 = (P.lg_gs == 4);
    Item<KIND, PTRS> it;
    // work item w: tile w / nm, 128-row block w % nm
    auto load_item = [&](uint32_t w) -> bool { return it.load(P, w / nm, w % nm, BN); };

    if (warp < LD_WARP0) {
        // -------------------------------------------------------- dequantisers
        const uint32_t r = tid & (BM - 1), h = tid >> 7;
        uint32_t g = 0;  // k-tiles of the CTA's earlier items: stage g % S, phase (g / S) & 1
        for (uint32_t i = 0;; i++) {
            uint32_t w;
            if (!next_item(i, true, w) || w >= n_items) break;
            if (!load_item(w)) continue;
            const size_t row_in = glu_row(tmin<uint32_t>(it.row0 + r, P.n - 1), GLU ? P.glu_nh : 0u);
            const uint8_t *srow = it.sb + row_in * P.groups * ES;
            const uint8_t *brow = it.bb + row_in * P.groups * 2u;
            const bool swords = PTRS ? it.ptr_scale_words : P.scale_words != 0;
            bool ok = true;
            for (uint32_t kt = 0; kt < P.ktiles; kt++, g++) {
                const uint32_t s = g % S;
                if (!ptx::mbar_wait_bounded(loaded0 + 8 * s, (g / S) & 1u, abort_flag, P.err, ERR_TIMEOUT,
                                            P.timeout_ns)) {
                    ok = false;
                    break;
                }
                const uint32_t st = base + s * STAGE;
                const uint8_t *stp = base_ptr + s * STAGE;
                if (BT == 2 && xmode == XM_LOADERS) {
                    // f32 x: elements 0-3 of a chunk landed in the hi tile's slot, 4-7 in the
                    // lo tile's slot; rewrite both as the bf16 hi and lo halves
                    const uint32_t cc = tid & 7u;
#pragma unroll
                    for (int j = 0; j < BN / 32; j++) {
                        const uint32_t i = (tid >> 3) + 32u * j;
                        if (i >= it.nt_pad) continue;
                        const uint32_t o = swz(i, cc);
                        const float4 v0 = *(const float4 *)(stp + B_OFF + o);
                        const float4 v1 = *(const float4 *)(stp + B_OFF + B_TILE + o);
                        const float f[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
                        uint32_t hi[4], lo[4];
#pragma unroll
                        for (int t = 0; t < 4; t++) {
                            hi[t] = pack2<false>(f[2 * t], f[2 * t + 1]);
                            const float2 hh = unpack2<false>(hi[t]);
                            lo[t] = pack2<false>(f[2 * t] - hh.x, f[2 * t + 1] - hh.y);
                        }
                        sts128(st + B_OFF + o, hi[0], hi[1], hi[2], hi[3]);
                        sts128(st + B_OFF + B_TILE + o, lo[0], lo[1], lo[2], lo[3]);
                    }
                }
                // this row's codes and scale words: the strided cp.async rows, or the TMA tile
                // (GLU: staged rows 0-63 hold the gate rows, 64-127 the up rows)
                const uint8_t *rr = stp + RAW_OFF + r * RL::STRIDE;
                const uint8_t *ct = stp + RAW_OFF;
                const uint32_t sr = GLU ? ((r & 1u) ? 64u + (r >> 1) : (r >> 1)) : r;
                const uint8_t *sw_row = tma ? ct + RL::TMA_SC + 16u * r : rr + RL::SC;
                uint32_t wv[Raw<KIND>::W];
                uint32_t sub = 0;
                uint32_t hw[16], lw[16];  // ATM: this thread's A words (hi and lo terms)
                if constexpr (KIND == K_AFF4 || KIND == K_CB4 || KIND == K_NVFP4 || KIND == K_MXFP4) {
                    const uint4 q = *(const uint4 *)(tma ? ct + tma_chunk<KIND>(sr, h) : rr + 16u * h);
                    wv[0] = q.x; wv[1] = q.y; wv[2] = q.z; wv[3] = q.w;
                } else if constexpr (KIND == K_AFF8) {
                    const uint4 q0 = *(const uint4 *)(tma ? ct + tma_chunk<KIND>(sr, 2u * h) : rr + 32u * h);
                    const uint4 q1 = *(const uint4 *)(tma ? ct + tma_chunk<KIND>(sr, 2u * h + 1u) : rr + 32u * h + 16u);
                    wv[0] = q0.x; wv[1] = q0.y; wv[2] = q0.z; wv[3] = q0.w;
                    wv[4] = q1.x; wv[5] = q1.y; wv[6] = q1.z; wv[7] = q1.w;
                } else if constexpr (KIND == K_AFF6) {
                    const uint8_t *cr = tma ? ct + sr * RL::RB : rr;
#pragma unroll
                    for (int i = 0; i < 3; i++) {
                        const uint2 q = *(const uint2 *)(cr + 24u * h + 8u * i);
                        wv[2 * i] = q.x; wv[2 * i + 1] = q.y;
                    }
                } else if constexpr (KIND == K_CB2) {
                    const uint2 q = *(const uint2 *)((tma ? ct + sr * RL::RB : rr) + 8u * h);
                    wv[0] = q.x; wv[1] = q.y;
                } else {  // K_CB3: codes from (kt*KT) % 10 + 32h of the window
                    const uint32_t c0 = (kt * KT) % 10u + 32u * h, wi = c0 / 10u;
                    sub = c0 - 10u * wi;
                    const uint8_t *cr = rr;
                    if (tma) {
                        // the row's window in the even- or odd-row copy, from its 16-byte start
                        const uint32_t odd = r & 1u, byte0 = odd * P.row_bytes + 4u * ((kt * KT) / 10u);
                        cr = ct + odd * (64u * CB3_WIN) + (r >> 1) * CB3_WIN + (byte0 & 15u);
                    }
#pragma unroll
                    for (int i = 0; i < 4; i++) wv[i] = *(const uint32_t *)(cr + 4u * (wi + i));
                }
                const uint32_t j0 = kt * KT, gh = (j0 + 32u * h) >> P.lg_gs;
                if constexpr (KIND == K_NVFP4) {
                    // groups of 16: this half's two E4M3 scales, converted together (exact in f16)
                    __half2 s01;
                    if (swords) {
                        // the staged word holds groups 4kt .. 4kt+3; this half's are bytes 2h, 2h+1
                        s01 = e4m3x2_to_half2((*(const uint32_t *)sw_row >> (16u * h)) & 0xFFFFu);
                    } else {
                        float s0, s1, unused;
                        global_scale<KIND>(srow, brow, gh, P.groups, s0, unused);
                        global_scale<KIND>(srow, brow, gh + 1u, P.groups, s1, unused);
                        s01 = __floats2half2_rn(s0, s1);
                    }
                    nvfp4_store<F16>(wv, s01, st, r, h * 4u);
                } else {
                    float s0, b0, s1 = 0.f, b1 = 0.f;
                    if (swords) {
                        const uint4 q = *(const uint4 *)sw_row;
                        const uint32_t sw[2] = {q.x, q.y}, bw[2] = {q.z, q.w};
                        const uint32_t base_b = ((j0 >> P.lg_gs) * ES) & ~3u;
                        staged_scale<KIND>(sw, bw, gh * ES - base_b, s0, b0);
                        if (gs16) staged_scale<KIND>(sw, bw, (gh + 1u) * ES - base_b, s1, b1);
                    } else {
                        global_scale<KIND>(srow, brow, gh, P.groups, s0, b0);
                        if (gs16) global_scale<KIND>(srow, brow, gh + 1u, P.groups, s1, b1);
                    }
                    if constexpr (CBF16) {
                        const __half2 h0 = __float2half2_rn(s0), h1 = __float2half2_rn(s1);  // exact: f16 scales
                        if constexpr (KIND == K_CB3) {
                            switch (sub) {  // first code's position in word 0: 0, 2, 4, 6 or 8
                                case 0: cb_pairs_f16<KIND, 0, ATM>(wv, h0, h1, gs16, lut2_s, st, st + A_TILE, r, h * 4u, hw, lw); break;
                                case 2: cb_pairs_f16<KIND, 2, ATM>(wv, h0, h1, gs16, lut2_s, st, st + A_TILE, r, h * 4u, hw, lw); break;
                                case 4: cb_pairs_f16<KIND, 4, ATM>(wv, h0, h1, gs16, lut2_s, st, st + A_TILE, r, h * 4u, hw, lw); break;
                                case 6: cb_pairs_f16<KIND, 6, ATM>(wv, h0, h1, gs16, lut2_s, st, st + A_TILE, r, h * 4u, hw, lw); break;
                                default: cb_pairs_f16<KIND, 8, ATM>(wv, h0, h1, gs16, lut2_s, st, st + A_TILE, r, h * 4u, hw, lw); break;
                            }
                        } else {
                            cb_pairs_f16<KIND, 0, ATM>(wv, h0, h1, gs16, lut2_s, st, st + A_TILE, r, h * 4u, hw, lw);
                        }
                    } else {
                        dequant_tile<KIND, F16, ATM>(wv, sub, s0, b0, s1, b1, gs16, cb_s, st, st + A_TILE, r, h * 4u,
                                                     hw, lw);
                    }
                }
                if constexpr (ATM) {
                    // this warp's 32 rows (its lane quarter), the thread's half of the k-tile
                    const uint32_t ta = tmem + ((32u * (warp & 3u)) << 16) + ACOL0 + s * (AT * A_TM_COLS) + h * 16u;
                    ptx::tmem_st16(ta, hw);
                    ptx::tmem_st16(ta + A_TM_COLS, lw);
                    ptx::tmem_wait_st();
                    ptx::tc_fence_before();
                    if (BT == 2 && xmode == XM_LOADERS) ptx::fence_proxy_async_smem();  // the rewritten B
                } else {
                    ptx::fence_proxy_async_smem();
                }
                ptx::mbar_arrive(full0 + 8 * s);
            }
            if (!ok) break;
        }
    } else if (warp < MMA_WARP) {
        // ------------------------------------------------------------- loaders
        const uint32_t lt = tid - NDQ;
        // x: thread lt copies 16-byte chunk lt % 8 of pair rows lt / 8 + XR j
        constexpr int NXL = BN * 8 / NLD;
        constexpr uint32_t XR = NLD / 8;  // pair rows per pass of the loaders
        constexpr uint32_t XS = (BT == 2) ? 4u : 2u;  // bytes per x element
        const uint32_t xc = lt & 7u, xi0 = lt >> 3;
        const uint32_t xdst0 = B_OFF + swz(xi0, xc);  // + XR * 128 j: XR rows further down
        const uint32_t nlast = P.n - 1;
        const uint32_t srow_bytes = P.groups * ES;
        const uint32_t nsw = (gs16 && ES == 2u) ? 2u : 1u;
        uint32_t g = 0;
        bool ok = true;
        for (uint32_t i = 0; ok; i++) {
            uint32_t w;
            if (!next_item(i, true, w) || w >= n_items) break;
            if (!load_item(w)) continue;
            const uint8_t *xrow[NXL];
#pragma unroll
            for (int j = 0; j < NXL; j++) {
                const uint32_t i = xi0 + XR * j;
                xrow[j] = (xmode == XM_LOADERS && i < it.nt)
                              ? (const uint8_t *)P.x +
                                    (size_t)(__ldg(P.sorted_pairs + it.off + it.r0 + i) / P.n_expert_used) * P.k * XS
                              : nullptr;
            }
            const uint8_t *ebase = it.wb;
            const uint32_t row0 = it.row0;
            // scale words: thread lt < BM stages those of weight row lt
            const size_t srow_in = glu_row(tmin<uint32_t>(row0 + (lt & (BM - 1)), nlast), GLU ? P.glu_nh : 0u);
            const uint8_t *srow = it.sb + srow_in * P.groups * ES;
            const uint8_t *brow = it.bb + srow_in * P.groups * 2u;
            const bool swords = PTRS ? it.ptr_scale_words : P.scale_words != 0;
            const bool raw16 = PTRS ? it.ptr_raw16 : P.raw16 != 0;
            for (uint32_t kt = 0; kt < P.ktiles; kt++, g++) {
                const uint32_t s = g % S;
                if (g >= S && !ptx::mbar_wait_bounded(empty0 + 8 * s, ((g / S) - 1u) & 1u, abort_flag, P.err,
                                                      ERR_TIMEOUT, P.timeout_ns)) {
                    ok = false;
                    break;
                }
                const uint32_t st = base + s * STAGE;
                // x rows of the pairs, straight into the B operand tile (zero past k and nt),
                // unless they come by tensor copy
                const uint32_t kk = kt * KT + xc * 8u;
#pragma unroll
                for (int j = 0; j < NXL; j++) {
                    if (xmode == XM_LOADERS && xi0 + XR * j < it.nt_pad) {
                        const bool in = xrow[j] != nullptr && kk < P.k;
                        const uint8_t *src = in ? xrow[j] + (size_t)kk * XS : (const uint8_t *)P.x;
                        const uint32_t dst = st + xdst0 + XR * 128u * j;
                        ptx::cp_async_16(dst, src, in ? 16u : 0u);
                        if constexpr (BT == 2) ptx::cp_async_16(dst + B_TILE, in ? src + 16 : src, in ? 16u : 0u);
                    }
                }
                // packed codes of the 128 rows (rows past n repeat row n-1; bytes past a row read as 0)
                const uint32_t raw = st + RAW_OFF;
                if (tma) {
                    // the codes come by tensor copy from the tensor-copy warp
                } else if constexpr (KIND == K_CB3) {
                    const uint32_t w0 = (kt * KT) / 10u;
#pragma unroll
                    for (int i = 0; i < BM * 8 / NLD; i++) {
                        const uint32_t q = lt + NLD * i, row = q >> 3, c = q & 7u;
                        const uint8_t *rp = ebase + (size_t)glu_row(tmin<uint32_t>(row0 + row, nlast), GLU ? P.glu_nh : 0u) * P.row_bytes;
                        const uint32_t o = (w0 + c) * 4u;
                        const bool in = o + 4u <= P.row_bytes;
                        ptx::cp_async_4(raw + row * RL::STRIDE + 4u * c, rp + (in ? o : 0u), in ? 4u : 0u);
                    }
                } else {
                    constexpr uint32_t RB = RL::RB;
                    if (raw16) {
                        constexpr uint32_t NC = RB / 16u;
#pragma unroll
                        for (uint32_t i = 0; i < (BM * NC + NLD - 1) / NLD; i++) {
                            const uint32_t q = lt + NLD * i, row = q / NC, c = q % NC;
                            if (row >= BM) break;
                            const uint8_t *rp = ebase + (size_t)glu_row(tmin<uint32_t>(row0 + row, nlast), GLU ? P.glu_nh : 0u) * P.row_bytes;
                            const uint32_t o = kt * RB + 16u * c;
                            const bool in = o < P.row_bytes;
                            ptx::cp_async_16(raw + row * RL::STRIDE + 16u * c, rp + (in ? o : 0u), in ? 16u : 0u);
                        }
                    } else {
                        constexpr uint32_t NC = RB / 8u;
#pragma unroll
                        for (uint32_t i = 0; i < (BM * NC + NLD - 1) / NLD; i++) {
                            const uint32_t q = lt + NLD * i, row = q / NC, c = q % NC;
                            if (row >= BM) break;
                            const uint8_t *rp = ebase + (size_t)glu_row(tmin<uint32_t>(row0 + row, nlast), GLU ? P.glu_nh : 0u) * P.row_bytes;
                            const uint32_t o = kt * RB + 8u * c;
                            const bool in = o < P.row_bytes;
                            ptx::cp_async_8(raw + row * RL::STRIDE + 8u * c, rp + (in ? o : 0u), in ? 8u : 0u);
                        }
                    }
                }
                if (swords && lt < BM) {
                    const uint32_t base_b = ((kt * KT >> P.lg_gs) * ES) & ~3u;
                    const uint32_t sdst = tma ? raw + RL::TMA_SC + 16u * lt : raw + lt * RL::STRIDE + RL::SC;
                    for (uint32_t i = 0; i < nsw; i++) {
                        const uint32_t o = base_b + 4u * i;
                        const bool in = o + 4u <= srow_bytes;
                        ptx::cp_async_4(sdst + 4u * i, srow + (in ? o : 0u), in ? 4u : 0u);
                        if constexpr (AFF) ptx::cp_async_4(sdst + 8u + 4u * i, brow + (in ? o : 0u), in ? 4u : 0u);
                    }
                }
                ptx::cp_async_mbar_arrive(loaded0 + 8 * s);
            }
        }
        ptx::cp_async_wait_all();
    } else if (warp == TMA_WARP) {
        // ------------------------------------------------------------ tensor copies
        if (lane == 0) {
            // per k-tile two 64-row copies of RB bytes per row (GLU: the 64 gate rows,
            // then the 64 up rows; rows past the expert's last read a neighbour's rows or
            // zeros and are never stored) and, for gathered x rows, the box of BN rows.
            // The arrival (with the byte count) is one of the stage's loaded arrivals.
            // Without tensor copies the lane only reads the ring.
            constexpr uint32_t RB = RL::RB;
            if (tma) ptx::prefetch_tensormap(&tmap);
            if (xmode == XM_ROWS) ptx::prefetch_tensormap(&xmap);
            // bytes per k-tile: the codes' two 64-row boxes, the x box of BN rows (each row
            // one 128-byte swizzle line; twice for f32 x)
            constexpr uint32_t CODE_TX = KIND == K_CB3 ? 2u * 64u * CB3_WIN : 2u * 64u * RB;
            const uint32_t tx0 = (tma ? CODE_TX : 0u) + (xmode == XM_ROWS ? (uint32_t)(BT * B_TILE) : 0u);
            const size_t img_tile = (size_t)P.ktiles * BN * 128u;
            uint32_t g = 0, last_s = 0, last_par = 0;
            bool any = false, ok = true;
            for (uint32_t i = 0; ok; i++) {
                uint32_t w;
                if (!next_item(i, false, w) || w >= n_items) break;
                if (!(tma || xmode != XM_LOADERS) || !load_item(w)) continue;
                // with the image: nt_pad lines of 128 bytes per k-tile
                const uint32_t tx = tx0 + (XIMG ? it.nt_pad * 128u : 0u);
                const uint8_t *img = XIMG ? P.ximage + (size_t)(w / nm) * img_tile : nullptr;
                const int32_t y0 = (int32_t)(it.e * P.n + (GLU ? it.row0 / 2u : it.row0));
                const int32_t y1 = GLU ? (int32_t)(it.e * P.n + P.glu_nh + it.row0 / 2u) : y0 + 64;
                for (uint32_t kt = 0; kt < P.ktiles; kt++, g++) {
                    const uint32_t s = g % S;
                    if (g >= S && !ptx::mbar_wait_bounded(empty0 + 8 * s, ((g / S) - 1u) & 1u, abort_flag, P.err,
                                                          ERR_TIMEOUT, P.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    const uint32_t bar = loaded0 + 8 * s, raw = base + s * STAGE + RAW_OFF;
                    ptx::mbar_arrive_expect_tx(bar, tx);
                    if (tma) {
                        if constexpr (KIND == K_CB3) {
                            // super-row (e n + row0) / 2 onwards: the even rows' window, then the odd rows'
                            const uint32_t byte0 = 4u * ((kt * KT) / 10u);
                            const int32_t ys = (int32_t)((it.e * P.n + it.row0) / 2u);
                            ptx::tma_load_2d(raw, &tmap, (int32_t)(byte0 & ~15u), ys, bar);
                            ptx::tma_load_2d(raw + 64u * CB3_WIN, &tmap, (int32_t)((P.row_bytes + byte0) & ~15u), ys, bar);
                        } else {
                            ptx::tma_load_2d(raw, &tmap, (int32_t)(kt * RB), y0, bar);
                            ptx::tma_load_2d(raw + 64u * RB, &tmap, (int32_t)(kt * RB), y1, bar);
                        }
                    }
                    if constexpr (XIMG)
                        ptx::bulk_g2s(base + s * STAGE + B_OFF, img + (size_t)kt * BN * 128u, it.nt_pad * 128u, bar);
                    if (xmode == XM_ROWS) {
                        // gathered rows off + r0 .. + BN - 1: rows past the tile's pairs are other
                        // pairs' x rows (or zeros past the end) in B rows whose results are not stored
                        const uint32_t xb = base + s * STAGE + B_OFF;
                        const int32_t xrow = (int32_t)(it.off + it.r0);
                        ptx::tma_load_2d(xb, &xmap, (int32_t)(kt * KT), xrow, bar);
                        if constexpr (BT == 2)
                            ptx::tma_load_2d(xb + B_TILE, &xmap, (int32_t)(kt * KT), xrow + (int32_t)P.xg_R, bar);
                    }
                    last_s = s;
                    last_par = (g / S) & 1u;
                    any = true;
                }
            }
            // copies still in flight after a wait gave up land before the CTA exits
            if (any) ptx::mbar_wait_bounded(loaded0 + 8 * last_s, last_par, nullptr, P.err, ERR_TIMEOUT, DRAIN_NS);
        }
    } else if (warp == MMA_WARP) {
        // --------------------------------------------------------------- MMA issue
        if (lane == 0) {
            bool ok = true;
            if (P.fault_ns) ok = ptx::mbar_wait_bounded(never, 0, abort_flag, P.err, ERR_TIMEOUT, P.fault_ns);
            uint32_t g = 0, done = 0;  // k-tiles consumed; items computed
            for (uint32_t i = 0; ok; i++) {
                uint32_t w;
                if (!next_item(i, false, w)) {
                    ok = false;
                    break;
                }
                if (w >= n_items) break;
                if (!load_item(w)) continue;
                const uint32_t buf = done % NACC, use = done / NACC;
                // the epilogue has read this accumulator's previous item (a fresh barrier's
                // preceding phase counts as complete, so the first two items do not wait)
                if (!ptx::mbar_wait_bounded(accempty0 + 8 * buf, (use & 1u) ^ 1u, abort_flag, P.err, ERR_TIMEOUT,
                                            P.timeout_ns)) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                const uint32_t d = tmem + buf * ACC_STRIDE;
                const uint32_t idesc = ptx::idesc_f16(F16 ? 0u : 1u, it.nt_pad);
                uint32_t accum = 0;
                for (uint32_t kt = 0; kt < P.ktiles; kt++, g++) {
                    const uint32_t s = g % S;
                    if (!ptx::mbar_wait_bounded(full0 + 8 * s, (g / S) & 1u, abort_flag, P.err, ERR_TIMEOUT,
                                                P.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    const uint32_t st = base + s * STAGE;
                    const uint32_t a_hi = st, a_lo = st + A_TILE;
                    const uint32_t b_hi = st + B_OFF, b_lo = b_hi + B_TILE;
#pragma unroll
                    for (int ks = 0; ks < KT / 16; ks++) {
                        const uint32_t ko = ks * 32u;
                        if constexpr (ATM) {
                            // 16 values of K: 8 columns of each A term
                            const uint32_t ta = tmem + ACOL0 + s * (AT * A_TM_COLS) + ks * 8u;
                            ptx::mma_f16_ts(d, ta, ptx::sdesc_k128(b_hi + ko), idesc, accum);
                            if constexpr (BT == 2) ptx::mma_f16_ts(d, ta, ptx::sdesc_k128(b_lo + ko), idesc, 1);
                            ptx::mma_f16_ts(d, ta + A_TM_COLS, ptx::sdesc_k128(b_hi + ko), idesc, 1);
                        } else {
                            ptx::mma_f16_ss(d, ptx::sdesc_k128(a_hi + ko), ptx::sdesc_k128(b_hi + ko), idesc, accum);
                            if constexpr (BT == 2)
                                ptx::mma_f16_ss(d, ptx::sdesc_k128(a_hi + ko), ptx::sdesc_k128(b_lo + ko), idesc, 1);
                            if constexpr (AT == 2)
                                ptx::mma_f16_ss(d, ptx::sdesc_k128(a_lo + ko), ptx::sdesc_k128(b_hi + ko), idesc, 1);
                        }
                        accum = 1;
                    }
                    ptx::mma_commit(empty0 + 8 * s);
                }
                if (!ok) break;
                ptx::mma_commit(accfull0 + 8 * buf);
                done++;
            }
            // every MMA issued has completed before TMEM is freed (its own limit, not the
            // pipeline waits' one)
            ptx::mma_commit(drainb);
            ptx::mbar_wait_bounded(drainb, 0, nullptr, P.err, ERR_TIMEOUT, DRAIN_NS);
        }
        __syncwarp();
    } else if (warp == SCHED_WARP) {
        // ------------------------------------------------------------- scheduler
        if (lane == 0) {
            for (uint32_t i = 0;; i++) {
                const uint32_t slot = i % RING;
                // every reader has taken the item published in this slot RING items ago
                if (i >= RING && !ptx::mbar_wait_bounded(ringempty0 + 8 * slot, ((i / RING) - 1u) & 1u, abort_flag,
                                                         P.err, ERR_TIMEOUT, P.timeout_ns))
                    break;
                uint32_t w = i == 0 ? blockIdx.x : gridDim.x + atomicAdd(P.work_counter, 1u);
                if (w > n_items) w = n_items;  // n_items: no more work
                ring[slot] = w;
                ptx::mbar_arrive(ringfull0 + 8 * slot);  // release: the item is visible to the readers
                if (w >= n_items) break;
            }
        }
    } else {
        // ------------------------------------------------------------- epilogue
        // TMEM -> registers (tcgen05.ld), times scale2 for NVFP4, plus the expert bias,
        // rounded once to the output type, stored to row p of out (the scatter back to
        // [token][slot] order). Warp w reads TMEM lanes 32 (w % 4) .. + 31.
        const uint32_t q = warp & 3u;
        uint32_t done = 0;
        for (uint32_t i = 0;; i++) {
            uint32_t w;
            if (!next_item(i, true, w) || w >= n_items) break;
            if (!load_item(w)) continue;
            const uint32_t buf = done % NACC, use = done / NACC;
            if (!ptx::mbar_wait_bounded(accfull0 + 8 * buf, use & 1u, abort_flag, P.err, ERR_TIMEOUT, P.timeout_ns))
                break;
            ptx::tc_fence_after();
            const uint32_t d = tmem + buf * ACC_STRIDE;
            const uint32_t grow_e = it.row0 + q * 32u + lane;  // logical row
            const uint32_t nh = GLU ? P.glu_nh : 0u;
            const float s2 = (KIND == K_NVFP4) ? __ldg((const float *)P.aux + it.e) : 1.f;
            const float bv =
                grow_e < P.n ? load_bias(P.bias, P.bias_dtype, (size_t)it.e * P.n + glu_row(grow_e, nh)) : 0.f;
            const uint32_t *pairs = P.sorted_pairs + it.off + it.r0;
            for (uint32_t c0 = 0; c0 < it.nt; c0 += 16) {
                uint32_t v[16], pr[16];
                ptx::tmem_ld16(d + ((q * 32u) << 16) + c0, v);
                // lane j < 16 fetches column c0 + j's pair (and its token's factor); the
                // warp shares them by shuffles
                const uint32_t cj = c0 + (lane & 15u);
                const uint32_t myp = cj < it.nt ? __ldg(pairs + cj) : 0u;
                const float myf = P.tok_scale ? __ldg(P.tok_scale + myp / P.n_expert_used) : 1.f;
#pragma unroll
                for (int i = 0; i < 16; i++) pr[i] = __shfl_sync(0xFFFFFFFFu, myp, i);
                ptx::tmem_wait_ld();
                if (P.tok_scale) {
                    // the token's factor (W4A4, or the power of two of the f16 image of bf16
                    // x), applied to the fp32 sum before the bias
#pragma unroll
                    for (int i = 0; i < 16; i++)
                        v[i] = __float_as_uint(__uint_as_float(v[i]) * __shfl_sync(0xFFFFFFFFu, myf, i));
                }
                if constexpr (GLU) {
                    // even lanes hold gate rows, the next lane the matching up row
#pragma unroll
                    for (int i = 0; i < 16; i++) {
                        const float y = __uint_as_float(v[i]) * s2 + bv;
                        const float up = __shfl_xor_sync(0xFFFFFFFFu, y, 1);
                        const uint32_t col = c0 + i;
                        if (col < it.nt && grow_e < P.n && !(lane & 1u))
                            store_out(P.out, P.out_dtype, (size_t)pr[i] * nh + (grow_e >> 1), glu_act(P.act, y) * up);
                    }
                } else if (grow_e < P.n) {
                    const uint32_t nc = tmin<uint32_t>(16u, it.nt - c0);
                    if (P.out_dtype == DT_BF16) {
#pragma unroll
                        for (int i = 0; i < 16; i++)
                            if ((uint32_t)i < nc)
                                ((__nv_bfloat16 *)P.out)[(size_t)pr[i] * P.n + grow_e] =
                                    __float2bfloat16_rn(__uint_as_float(v[i]) * s2 + bv);
                    } else {
#pragma unroll
                        for (int i = 0; i < 16; i++)
                            if ((uint32_t)i < nc)
                                store_out(P.out, P.out_dtype, (size_t)pr[i] * P.n + grow_e, __uint_as_float(v[i]) * s2 + bv);
                    }
                }
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(accempty0 + 8 * buf);
            done++;
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == MMA_WARP) {
        __syncwarp();
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, TMEM_COLS);
    }
}

// Dynamic shared memory per CTA (stages + 1 KB for aligning them), leaving room
// for the kernel's static shared memory within the 227 KB a CTA may use.
constexpr size_t GEMM_SMEM_BUDGET = 229000;

struct GemmPlan {
    uint32_t bn;
    int stages;
    size_t smem;
};

uint32_t raw_tile(int kind) {
    switch (kind) {
        case K_AFF4: return RawLayout<K_AFF4>::TILE;
        case K_AFF6: return RawLayout<K_AFF6>::TILE;
        case K_AFF8: return RawLayout<K_AFF8>::TILE;
        case K_CB2: return RawLayout<K_CB2>::TILE;
        case K_CB3: return RawLayout<K_CB3>::TILE;
        case K_CB4: return RawLayout<K_CB4>::TILE;
        case K_MXFP4: return RawLayout<K_MXFP4>::TILE;
        default: return RawLayout<K_NVFP4>::TILE;
    }
}

// Tile width and pipeline depth: when experts hold ~100 or more pairs on
// average, 256 pairs per tile (128 with f32 x, whose operand tiles are twice
// as large), so that two TMEM accumulators of the tile width fit the 512 columns
// and an item's epilogue overlaps the next item's MMAs; 64 otherwise. As many
// stages (2..6) as fit in one CTA per SM.
bool gemm_plan(const QmmArgs &a, GemmPlan *pl) {
    const uint64_t R = (uint64_t)a.m * a.n_expert_used;
    const bool big = R >= 96ull * a.num_experts;
    const bool f32x = a.x_dtype == DT_F32;
    const bool fp4 = a.kind == K_NVFP4 || a.kind == K_MXFP4;  // single-term A
    const uint32_t bn = big ? (f32x ? 128u : 256u) : 64u;
    const uint32_t at = fp4 ? 1u : 2u, bt = f32x ? 2u : 1u;
    const bool atm = at == 2u && bn <= 128u;  // A in tensor memory (GemmCfg::ATM)
    const size_t stage = (atm ? 0u : (size_t)at * A_TILE) + (size_t)bt * bn * KT * 2 + raw_tile(a.kind);
    if (2 * stage + 1024 > GEMM_SMEM_BUDGET) return false;
    int S = (int)((GEMM_SMEM_BUDGET - 1024) / stage);
    S = S > MAX_STAGES ? MAX_STAGES : S;
    if (atm) {  // the A terms of every stage beside the two accumulators in 512 columns
        const int s_tm = (int)((512u - 2u * bn) / (at * A_TM_COLS));
        S = S > s_tm ? s_tm : S;
    }
    pl->bn = bn;
    pl->stages = S;
    pl->smem = (size_t)S * stage + 1024;
    return true;
}

// Streaming multiprocessors of the current device (cached per device).
uint32_t sm_count_gemm() {
    static int count[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148u;
    if (count[dev] == 0) {
        int c = 0;
        if (cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || c <= 0) c = 148;
        count[dev] = c;
    }
    return (uint32_t)count[dev];
}

template <int KIND, int XT, int BN, bool PTRS, bool GLU, bool XIMG = false>
cudaError_t launch_tp(const GemmParams &P0, const CUtensorMap &tmap, const CUtensorMap &xmap, const GemmPlan &pl,
                      uint32_t n_mtiles, uint32_t max_tiles, cudaStream_t st) {
    GemmParams P = P0;
    P.stages = (uint32_t)pl.stages;
    auto kern = grouped_gemm_kernel<KIND, XT, BN, PTRS, GLU, XIMG>;
    static int smem_set[64];
    cudaError_t e = ensure_dyn_smem(kern, pl.smem, smem_set);
    if (e != cudaSuccess) return e;
    // persistent: one CTA per SM, or fewer when there are fewer work items
    const uint64_t items = (uint64_t)n_mtiles * max_tiles;
    const uint32_t ctas = (uint32_t)(items < (uint64_t)sm_count_gemm() ? items : (uint64_t)sm_count_gemm());
    kern<<<ctas, GEMM_THREADS, pl.smem, st>>>(P, tmap, xmap);
    return cudaGetLastError();
}

template <int KIND, int XT, int BN>
cudaError_t launch_t(const GemmParams &P, const CUtensorMap &tm, const CUtensorMap &xm, const GemmPlan &pl,
                     uint32_t n_mtiles, uint32_t max_tiles, cudaStream_t st) {
    if (P.packed_ptrs) return launch_tp<KIND, XT, BN, true, false>(P, tm, xm, pl, n_mtiles, max_tiles, st);
    if (P.glu_nh) return launch_tp<KIND, XT, BN, false, true>(P, tm, xm, pl, n_mtiles, max_tiles, st);
    if constexpr (XT == DT_F16) {
        if (P.xmode == XM_IMAGE) return launch_tp<KIND, XT, BN, false, false, true>(P, tm, xm, pl, n_mtiles, max_tiles, st);
    }
    return launch_tp<KIND, XT, BN, false, false>(P, tm, xm, pl, n_mtiles, max_tiles, st);
}

template <int KIND>
cudaError_t launch_k(const GemmParams &P, const CUtensorMap &tm, const CUtensorMap &xm, const GemmPlan &pl,
                     int x_dtype, uint32_t nm, uint32_t mt, cudaStream_t st) {
    if (x_dtype == DT_F32) {
        if (pl.bn == 128) return launch_t<KIND, DT_F32, 128>(P, tm, xm, pl, nm, mt, st);
        return launch_t<KIND, DT_F32, 64>(P, tm, xm, pl, nm, mt, st);
    }
    if constexpr (KIND == K_MXFP4) {
        // e2m1 * 2^e can leave the f16 range: only bf16 (and f32, as bf16 halves) x here
        if (x_dtype != DT_BF16) return cudaErrorNotSupported;
        if (pl.bn == 256) return launch_t<KIND, DT_BF16, 256>(P, tm, xm, pl, nm, mt, st);
        return launch_t<KIND, DT_BF16, 64>(P, tm, xm, pl, nm, mt, st);
    } else {
    if (x_dtype == DT_BF16) {
        if (pl.bn == 256) return launch_t<KIND, DT_BF16, 256>(P, tm, xm, pl, nm, mt, st);
        return launch_t<KIND, DT_BF16, 64>(P, tm, xm, pl, nm, mt, st);
    }
    if (pl.bn == 256) return launch_t<KIND, DT_F16, 256>(P, tm, xm, pl, nm, mt, st);
    return launch_t<KIND, DT_F16, 64>(P, tm, xm, pl, nm, mt, st);
    }
}

cudaError_t launch_kind(const GemmParams &P, const CUtensorMap &tm, const CUtensorMap &xm, const GemmPlan &pl,
                        int kind, int x_dtype, uint32_t nm, uint32_t mt, cudaStream_t st) {
    switch (kind) {
        case K_AFF4: return launch_k<K_AFF4>(P, tm, xm, pl, x_dtype, nm, mt, st);
        case K_AFF6: return launch_k<K_AFF6>(P, tm, xm, pl, x_dtype, nm, mt, st);
        case K_AFF8: return launch_k<K_AFF8>(P, tm, xm, pl, x_dtype, nm, mt, st);
        case K_CB2: return launch_k<K_CB2>(P, tm, xm, pl, x_dtype, nm, mt, st);
        case K_CB3: return launch_k<K_CB3>(P, tm, xm, pl, x_dtype, nm, mt, st);
        case K_CB4: return launch_k<K_CB4>(P, tm, xm, pl, x_dtype, nm, mt, st);
        case K_NVFP4: return launch_k<K_NVFP4>(P, tm, xm, pl, x_dtype, nm, mt, st);
        case K_MXFP4: return launch_k<K_MXFP4>(P, tm, xm, pl, x_dtype, nm, mt, st);
        default: return cudaErrorInvalidValue;
    }
}

// cuTensorMapEncodeTiled, looked up once through the runtime (null if unavailable).
PFN_cuTensorMapEncodeTiled_v12000 encode_tiled() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = []() -> PFN_cuTensorMapEncodeTiled_v12000 {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        return (PFN_cuTensorMapEncodeTiled_v12000)f;
    }();
    return fn;
}

// Bytes of one k-tile of one packed row (the staging's RB) for each storage kind.
uint32_t ktile_row_bytes(int kind) {
    switch (kind) {
        case K_AFF4: return RawLayout<K_AFF4>::RB;
        case K_AFF6: return RawLayout<K_AFF6>::RB;
        case K_AFF8: return RawLayout<K_AFF8>::RB;
        case K_CB2: return RawLayout<K_CB2>::RB;
        case K_CB4: return RawLayout<K_CB4>::RB;
        case K_NVFP4: return RawLayout<K_NVFP4>::RB;
        case K_MXFP4: return RawLayout<K_MXFP4>::RB;
        default: return 0;
    }
}

// Tensor map of rows of 16-bit x values, a [rows, k] matrix, with boxes of 64
// values x box_rows rows in the 128-byte swizzle (the B operand's canonical
// K-major layout). False if it cannot be encoded.
bool x_tensor_map(const void *x, uint32_t rows, uint32_t k, uint32_t box_rows, CUtensorMap *m) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = encode_tiled();
    if (!enc || (uintptr_t)x % 16u != 0 || k % 8u != 0 || box_rows == 0 || box_rows > 256u || rows == 0) return false;
    const cuuint64_t dims[2] = {k, rows};
    const cuuint64_t strides[1] = {(cuuint64_t)k * 2u};
    const cuuint32_t box[2] = {64u, box_rows};
    const cuuint32_t estr[2] = {1u, 1u};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, (void *)x, dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tensor map of the packed codes as a [num_experts * n, row_bytes] byte matrix with
// 64-row x RB-byte boxes, swizzled as tma_chunk expects. False when the codes
// cannot be staged this way (pointer tables, 3-bit rows, rows not a multiple of
// 16 bytes, or no driver entry point).
bool code_tensor_map(const QmmArgs &a, CUtensorMap *m) {
    const uint64_t rows = (uint64_t)a.num_experts * a.n;
    if (a.packed_ptrs || (uintptr_t)a.packed % 16u != 0 || rows >= (1ull << 31)) return false;
    PFN_cuTensorMapEncodeTiled_v12000 enc = encode_tiled();
    if (!enc) return false;
    if (a.kind == K_CB3) {
        // super-rows of two rows (a multiple of 16 bytes when a row is of 8), never
        // straddling two experts (n even); not with a gated output, whose A tiles
        // pair rows from the two halves
        if (a.row_bytes % 8u != 0 || a.n % 2u != 0 || a.act >= 0) return false;
        const cuuint64_t dims[2] = {2ull * a.row_bytes, rows / 2};
        const cuuint64_t strides[1] = {2ull * a.row_bytes};
        const cuuint32_t box[2] = {CB3_WIN, 64u};
        const cuuint32_t estr[2] = {1u, 1u};
        return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, (void *)a.packed, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
    }
    const uint32_t rb = ktile_row_bytes(a.kind);
    if (!rb || a.row_bytes % 16u != 0) return false;
    const cuuint64_t dims[2] = {a.row_bytes, rows};
    const cuuint64_t strides[1] = {a.row_bytes};
    const cuuint32_t box[2] = {rb, 64u};
    const cuuint32_t estr[2] = {1u, 1u};
    const CUtensorMapSwizzle sw = rb == 32u ? CU_TENSOR_MAP_SWIZZLE_32B
                                : rb == 64u ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_NONE;
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, (void *)a.packed, dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool gemm_supported(const QmmArgs &a) {
    // MXFP4 weights e2m1 * 2^e are exact in bf16 but can leave the f16 range: f16 x
    // stays on the CUDA-core paths
    if (a.kind == K_MXFP4 && a.x_dtype == DT_F16) return false;
    const uint32_t gs = a.group_size;
    if (gs < 16 || (gs & (gs - 1)) != 0) return false;
    if (a.k % 8 != 0 || a.k % gs != 0) return false;
    // packed codes are staged with 8- or 16-byte copies (4-byte words for 3-bit codebook rows)
    if (a.row_bytes % (a.kind == K_CB3 ? 4u : 8u) != 0) return false;
    if ((uintptr_t)a.packed % 16 != 0 || (uintptr_t)a.x % 16 != 0) return false;
    if (a.num_experts > ROUTE_MAX_E) return false;
    GemmPlan pl;
    return gemm_plan(a, &pl);
}

uint32_t gemm_tile_rows(const QmmArgs &a) {
    GemmPlan pl;
    return gemm_plan(a, &pl) ? pl.bn : 64u;
}

cudaError_t launch_gemm(const QmmArgs &a, const uint32_t *offsets, const uint32_t *sorted_pairs,
                        const uint32_t *tiles, const uint32_t *tile_count, uint32_t max_tiles,
                        uint32_t *err, uint32_t *work_counter, const uint16_t *xg, const uint8_t *ximg,
                        cudaStream_t st) {
    GemmPlan pl;
    if (!gemm_plan(a, &pl)) return cudaErrorNotSupported;
    GemmParams P{};
    P.x = a.x; P.offsets = offsets; P.sorted_pairs = sorted_pairs; P.tiles = tiles;
    P.tile_count = tile_count; P.packed = a.packed; P.scales = a.scales; P.aux = a.aux;
    P.out = a.out; P.err = err;
    P.k = a.k; P.n = a.n;
    uint32_t lg = 0;
    while ((1u << lg) < a.group_size) lg++;
    P.lg_gs = lg;
    P.groups = a.groups; P.n_expert_used = a.n_expert_used; P.row_bytes = a.row_bytes;
    P.ktiles = (a.k + KT - 1) / KT;
    const uint32_t es = (a.kind == K_NVFP4 || a.kind == K_MXFP4) ? 1u : 2u;
    P.scale_words = (a.groups * es) % 4u == 0 && (uintptr_t)a.scales % 4u == 0 &&
                    (a.fmt != FMT_AFFINE || (uintptr_t)a.aux % 4u == 0);
    P.raw16 = a.kind != K_CB3 && a.row_bytes % 16u == 0;
    P.out_dtype = a.out_dtype;
    P.bias = a.bias; P.bias_dtype = a.bias_dtype;
    P.packed_ptrs = a.packed_ptrs; P.scale_ptrs = a.scale_ptrs; P.bias_ptrs = a.bias_ptrs;
    P.timeout_ns = WAIT_NS;
    P.fault_ns = a.fault_wait_ns;
    P.glu_nh = a.act >= 0 ? a.n / 2u : 0u;
    P.act = a.act;
    CUtensorMap tmap;
    memset(&tmap, 0, sizeof(tmap));
    P.tma = code_tensor_map(a, &tmap) ? 1u : 0u;
    const uint32_t nm = (a.n + BM - 1) / BM;
    P.n_mtiles = nm;
    P.work_counter = work_counter;
    CUtensorMap xmap;
    memset(&xmap, 0, sizeof(xmap));
    const uint32_t R = a.m * a.n_expert_used;
    P.xg_R = R;
    P.tok_scale = a.tok_scale;
    // f32 x: tensor copies of the rows gathered and split after routing, when the
    // workspace holds them (and no test asks for the loader copies)
    P.xmode = (a.x_dtype == DT_F32 && !a.x_copies && xg && x_tensor_map(xg, R * 2u, a.k, pl.bn, &xmap))
                  ? XM_ROWS
                  : XM_LOADERS;
    // 16-bit x as the f16 image (the caller sets a.x_dtype to f16 with it)
    P.ximage = nullptr;
    if (ximg && a.x_dtype == DT_F16 && !a.packed_ptrs && a.act < 0) {
        P.xmode = XM_IMAGE;
        P.ximage = ximg;
    }
    return launch_kind(P, tmap, xmap, pl, a.kind, a.x_dtype, nm, max_tiles, st);
}

}  // namespace moe
