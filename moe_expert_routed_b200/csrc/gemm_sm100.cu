// gemm_sm100.cu -- expert-grouped GEMM on the 5th-generation tensor cores (tcgen05).
//
// One CTA computes a 128 x BN tile of one expert: 128 consecutive weight rows
// (output columns) of expert e against up to BN of the (token, slot) pairs
// routed to e (a tile of the routing prologue's tile list). Operands are
// swapped relative to out = x * W^T: the dequantised weight tile is the MMA's
// A operand (M = 128) and the gathered token rows are B (N = pairs in the tile,
// rounded up to 16), so each weight tile is dequantised once per tile of pairs.
// The pages' designs that this replaces: fused Metal dequant to fp16 followed
// by gather_mm (turboquant fast_switch_patch.py) and the routed W4A16 grouped
// GEMM fed by expert_offsets / sorted_token_ids (metrale helpers_b.rs,
// launch_grouped_gemm).
//
// Warp roles (288 threads):
//   warps 0-7  producers: per 64-wide k-tile, dequantise 128 rows x 64 codes to
//              16-bit values in the 128-byte-swizzled K-major layout and gather
//              the pairs' x rows (cp.async, or f32 loads split into two bf16
//              halves); then the epilogue: TMEM -> registers (tcgen05.ld),
//              times scale2 for NVFP4, rounded once to the output type, stored to
//              row p of out (the scatter back to [token][slot] order).
//   warp 8     TMEM allocation; one lane issues tcgen05.mma (kind::f16, fp32
//              accumulation in TMEM) and tcgen05.commit.
// Stages are handed over with mbarriers (full: 256 producer arrivals; empty and
// accumulator-ready: tcgen05.commit). Every wait is bounded (1 s); a wait that
// gives up sets ERR_TIMEOUT, the CTA drains its in-flight MMAs and copies,
// frees TMEM and exits.
//
// Exactness: products must stay exact so that the fp32 accumulation is the
// only rounding. NVFP4 weights e2m1 * e4m3 have at most 6 significant bits and
// are exact in bf16/f16: one MMA per k-step. Affine (c*s + b) and codebook
// (cb[c]*s) weights are formed in fp32 and split into a 16-bit high part and
// the 16-bit rounding of the remainder (two MMAs). f32 x is split the same way
// into two bf16 halves; the lo*lo product is dropped (below 2^-16 relative).
#include "common.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace moe {

namespace {

constexpr int BM = 128;
constexpr int KT = 64;  // k per tile: one 128-byte swizzle atom of 16-bit values
constexpr int NPROD = 256;
constexpr int GEMM_THREADS = NPROD + 32;
constexpr int MMA_WARP = NPROD / 32;
constexpr int A_TILE = BM * KT * 2;  // bytes per A term per stage
constexpr uint64_t WAIT_NS = 1000000000ull;

struct GemmParams {
    const void *x;
    const uint32_t *offsets, *sorted_pairs, *tiles, *tile_count;
    const uint8_t *packed;
    const void *scales;
    const void *aux;
    void *out;
    uint32_t *err;
    uint32_t k, n, lg_gs, groups, n_expert_used, row_bytes, ktiles, stages;
    int out_dtype;
    uint64_t timeout_ns;
};

template <int KIND> constexpr int a_terms() { return KIND == K_NVFP4 ? 1 : 2; }

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

template <bool F16>
__device__ __forceinline__ float round16(float v) {
    if constexpr (F16) return __half2float(__float2half_rn(v));
    else return __bfloat162float(__float2bfloat16_rn(v));
}

__device__ __forceinline__ uint2 ldg64_guard(const uint8_t *row, uint32_t off, uint32_t row_bytes) {
    if (off + 8u <= row_bytes) return __ldg((const uint2 *)(row + off));
    return make_uint2(0u, 0u);
}

// Raw words holding codes [j0, j0+32) of one row (j0 a multiple of 32).
template <int KIND> struct Raw;
template <> struct Raw<K_AFF4> { static constexpr int W = 4; };
template <> struct Raw<K_CB4> { static constexpr int W = 4; };
template <> struct Raw<K_NVFP4> { static constexpr int W = 4; };
template <> struct Raw<K_AFF8> { static constexpr int W = 8; };
template <> struct Raw<K_AFF6> { static constexpr int W = 6; };
template <> struct Raw<K_CB2> { static constexpr int W = 2; };
template <> struct Raw<K_CB3> { static constexpr int W = 5; };

template <int KIND>
__device__ __forceinline__ void load_raw(const uint8_t *row, uint32_t j0, uint32_t row_bytes,
                                         uint32_t (&w)[Raw<KIND>::W], uint32_t &sub) {
    sub = 0;
    if constexpr (KIND == K_CB3) {
        const uint32_t w0 = j0 / 10u;
        sub = j0 - 10u * w0;
#pragma unroll
        for (int i = 0; i < 5; i++) {
            const uint32_t off = (w0 + i) * 4u;
            w[i] = (off + 4u <= row_bytes) ? __ldg((const uint32_t *)(row + off)) : 0u;
        }
    } else {
        constexpr int BITS = kind_bits(KIND);
        const uint32_t off = j0 * BITS / 8u;  // multiple of 8 bytes
#pragma unroll
        for (int i = 0; i < Raw<KIND>::W / 2; i++) {
            uint2 v = ldg64_guard(row, off + 8u * i, row_bytes);
            w[2 * i] = v.x;
            w[2 * i + 1] = v.y;
        }
    }
}

template <int KIND, int I>
__device__ __forceinline__ uint32_t raw_code(const uint32_t (&w)[Raw<KIND>::W], uint32_t sub) {
    if constexpr (KIND == K_AFF4 || KIND == K_CB4 || KIND == K_NVFP4) {
        return (w[I / 8] >> (4 * (I % 8))) & 15u;
    } else if constexpr (KIND == K_AFF8) {
        return (w[I / 4] >> (8 * (I % 4))) & 255u;
    } else if constexpr (KIND == K_CB2) {
        return (w[I / 16] >> (2 * (I % 16))) & 3u;
    } else if constexpr (KIND == K_AFF6) {
        constexpr int b = 6 * I, wi = b / 32, sh = b % 32;
        if constexpr (sh <= 26) return (w[wi] >> sh) & 63u;
        else return __funnelshift_r(w[wi], w[wi + 1], sh) & 63u;
    } else {  // K_CB3: code (sub + I) of the 5 loaded words, 10 codes per word
        const uint32_t idx = sub + I;
        const uint32_t wi = (idx * 205u) >> 11;  // idx / 10 for idx < 1029
        const uint32_t sh = 3u * (idx - 10u * wi);
        const uint32_t word = wi == 0 ? w[0] : wi == 1 ? w[1] : wi == 2 ? w[2] : wi == 3 ? w[3] : w[4];
        return (word >> sh) & 7u;
    }
}

template <int KIND, int I>
struct DeqLoop {
    static __device__ __forceinline__ void run(const uint32_t (&w)[Raw<KIND>::W], uint32_t sub,
                                               float s0, float b0, float s1, float b1,
                                               bool two_groups, const float *cb, float (&v)[32]) {
        if constexpr (I < 32) {
            const uint32_t code = raw_code<KIND, I>(w, sub);
            const float s = (I >= 16 && two_groups) ? s1 : s0;
            const float b = (I >= 16 && two_groups) ? b1 : b0;
            if constexpr (KIND == K_AFF4 || KIND == K_AFF6 || KIND == K_AFF8) v[I] = fmaf((float)code, s, b);
            else if constexpr (KIND == K_NVFP4) v[I] = e2m1_to_f32(code) * s;
            else v[I] = cb[code] * s;
            DeqLoop<KIND, I + 1>::run(w, sub, s0, b0, s1, b1, two_groups, cb, v);
        }
    }
};

// Dequantise the thread's 32 codes and store them as 4 chunks of 8 16-bit values
// (hi term, and lo term when present) at chunk positions c0 .. c0+3 of row r.
template <int KIND, bool F16>
__device__ __forceinline__ void dequant_store(const uint32_t (&w)[Raw<KIND>::W], uint32_t sub,
                                              float s0, float b0, float s1, float b1, bool two_groups,
                                              const float *cb, uint32_t a_hi, uint32_t a_lo,
                                              uint32_t r, uint32_t c0) {
    float v[32];
    DeqLoop<KIND, 0>::run(w, sub, s0, b0, s1, b1, two_groups, cb, v);
#pragma unroll
    for (int cc = 0; cc < 4; cc++) {
        uint32_t h[4], l[4];
#pragma unroll
        for (int e = 0; e < 4; e++) {
            const float x0 = v[cc * 8 + 2 * e], x1 = v[cc * 8 + 2 * e + 1];
            h[e] = pack2<F16>(x0, x1);
            if constexpr (a_terms<KIND>() == 2)
                l[e] = pack2<F16>(x0 - round16<F16>(x0), x1 - round16<F16>(x1));
        }
        const uint32_t off = swz(r, c0 + cc);
        sts128(a_hi + off, h[0], h[1], h[2], h[3]);
        if constexpr (a_terms<KIND>() == 2) sts128(a_lo + off, l[0], l[1], l[2], l[3]);
    }
}

template <int KIND>
__device__ __forceinline__ void load_scales(const GemmParams &P, size_t row_index, uint32_t g,
                                            float &s, float &b) {
    g = min(g, P.groups - 1u);
    const size_t i = row_index * P.groups + g;
    if constexpr (KIND == K_AFF4 || KIND == K_AFF6 || KIND == K_AFF8) {
        s = bf16_bits_to_f32(__ldg((const unsigned short *)P.scales + i));
        b = bf16_bits_to_f32(__ldg((const unsigned short *)P.aux + i));
    } else if constexpr (KIND == K_NVFP4) {
        s = e4m3_to_f32(__ldg((const uint8_t *)P.scales + i));
        b = 0.f;
    } else {
        s = f16_bits_to_f32(__ldg((const unsigned short *)P.scales + i));
        b = 0.f;
    }
}

template <int KIND, int XT, int BN>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
grouped_gemm_kernel(const GemmParams P) {
    constexpr int AT = a_terms<KIND>();
    constexpr int BT = (XT == DT_F32) ? 2 : 1;
    constexpr bool F16 = (XT == DT_F16);
    constexpr int B_TILE = BN * KT * 2;
    constexpr int STAGE = AT * A_TILE + BT * B_TILE;

    extern __shared__ uint8_t smem_raw[];
    __shared__ uint64_t bars[2 * 8 + 1];
    __shared__ uint32_t tmem_s;
    __shared__ int abort_s;
    __shared__ uint32_t pairs_s[BN];
    __shared__ uint32_t tok_s[BN];
    __shared__ float cb_s[16];

    const uint32_t tile = blockIdx.y;
    if (tile >= __ldg(P.tile_count)) return;  // uniform
    const uint32_t tid = threadIdx.x, warp = tid >> 5, lane = tid & 31u;
    const uint32_t e = __ldg(P.tiles + 2 * tile), r0 = __ldg(P.tiles + 2 * tile + 1);
    const uint32_t off = __ldg(P.offsets + e);
    const uint32_t cnt = __ldg(P.offsets + e + 1) - off;
    const uint32_t nt = tmin<uint32_t>(BN, cnt - r0);
    const uint32_t nt_pad = (nt + 15u) & ~15u;
    const uint32_t row0 = blockIdx.x * BM;
    const uint32_t S = P.stages;

    const uint32_t base = (ptx::smem_u32(smem_raw) + 1023u) & ~1023u;
    const uint32_t full0 = ptx::smem_u32(&bars[0]);
    const uint32_t empty0 = ptx::smem_u32(&bars[8]);
    const uint32_t accb = ptx::smem_u32(&bars[16]);
    volatile int *abort_flag = &abort_s;

    if (tid == 0) {
        for (uint32_t s = 0; s < S; s++) {
            ptx::mbar_init(full0 + 8 * s, NPROD);
            ptx::mbar_init(empty0 + 8 * s, 1);
        }
        ptx::mbar_init(accb, 1);
        ptx::fence_mbar_init();
        abort_s = 0;
    }
    for (uint32_t i = tid; i < BN; i += blockDim.x) {
        const uint32_t p = i < nt ? __ldg(P.sorted_pairs + off + r0 + i) : 0u;
        pairs_s[i] = p;
        tok_s[i] = p / P.n_expert_used;
    }
    if constexpr (KIND == K_CB2 || KIND == K_CB3 || KIND == K_CB4) {
        if (tid < (1u << kind_bits(KIND)))
            cb_s[tid] = f16_bits_to_f32(__ldg((const unsigned short *)P.aux + tid));
    }
    if (warp == MMA_WARP) {
        ptx::tmem_alloc(ptx::smem_u32(&tmem_s), BN);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = tmem_s;

    if (warp < MMA_WARP) {
        // ------------------------------------------------------------ producers
        const uint32_t r = tid & (BM - 1), h = tid >> 7;
        const uint32_t grow = row0 + r;
        const uint32_t growc = grow < P.n ? grow : P.n - 1;
        const size_t row_index = (size_t)e * P.n + growc;
        const uint8_t *rowp = P.packed + row_index * P.row_bytes;
        const bool gs16 = (P.lg_gs == 4);
        bool ok = true;
        for (uint32_t kt = 0; kt < P.ktiles; kt++) {
            const uint32_t s = kt % S, use = kt / S;
            if (use > 0 && !ptx::mbar_wait_bounded(empty0 + 8 * s, (use - 1) & 1u, abort_flag,
                                                   P.err, ERR_TIMEOUT, P.timeout_ns)) {
                ok = false;
                break;
            }
            const uint32_t st = base + s * STAGE;
            const uint32_t b_hi = st + AT * A_TILE;
            // gather x rows of the pairs: token i, 16-byte chunk c of this k-tile
            if constexpr (BT == 1) {
                for (uint32_t q = tid; q < nt_pad * 8u; q += NPROD) {
                    const uint32_t i = q >> 3, c = q & 7u;
                    const uint32_t kk = kt * KT + c * 8u;
                    const bool in = i < nt && kk < P.k;
                    const uint16_t *src = (const uint16_t *)P.x + (in ? (size_t)tok_s[i] * P.k + kk : 0);
                    ptx::cp_async_16(b_hi + swz(i, c), src, in ? 16u : 0u);
                }
                ptx::cp_async_commit();
            } else {
                const uint32_t b_lo = b_hi + B_TILE;
                for (uint32_t q = tid; q < nt_pad * 8u; q += NPROD) {
                    const uint32_t i = q >> 3, c = q & 7u;
                    const uint32_t kk = kt * KT + c * 8u;
                    float4 v0 = make_float4(0.f, 0.f, 0.f, 0.f), v1 = v0;
                    if (i < nt && kk < P.k) {
                        const float4 *src = (const float4 *)((const float *)P.x + (size_t)tok_s[i] * P.k + kk);
                        v0 = __ldg(src);
                        v1 = __ldg(src + 1);
                    }
                    const float f[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
                    uint32_t hi[4], lo[4];
#pragma unroll
                    for (int t = 0; t < 4; t++) {
                        hi[t] = pack2<false>(f[2 * t], f[2 * t + 1]);
                        lo[t] = pack2<false>(f[2 * t] - round16<false>(f[2 * t]),
                                             f[2 * t + 1] - round16<false>(f[2 * t + 1]));
                    }
                    const uint32_t o = swz(i, c);
                    sts128(b_hi + o, hi[0], hi[1], hi[2], hi[3]);
                    sts128(b_lo + o, lo[0], lo[1], lo[2], lo[3]);
                }
            }
            // dequantise this thread's 32 codes of row r
            {
                const uint32_t j0 = kt * KT + h * 32u;
                uint32_t w[Raw<KIND>::W];
                uint32_t sub;
                load_raw<KIND>(rowp, j0, P.row_bytes, w, sub);
                float s0, b0, s1 = 0.f, b1 = 0.f;
                load_scales<KIND>(P, row_index, j0 >> P.lg_gs, s0, b0);
                if (gs16) load_scales<KIND>(P, row_index, (j0 >> 4) + 1u, s1, b1);
                dequant_store<KIND, F16>(w, sub, s0, b0, s1, b1, gs16, cb_s, st, st + A_TILE, r,
                                         h * 4u);
            }
            if constexpr (BT == 1) ptx::cp_async_wait_all();
            ptx::fence_proxy_async_smem();
            ptx::mbar_arrive(full0 + 8 * s);
        }
        if (!ok) ptx::cp_async_wait_all();
        // ------------------------------------------------------------- epilogue
        if (ok && ptx::mbar_wait_bounded(accb, 0, abort_flag, P.err, ERR_TIMEOUT, P.timeout_ns)) {
            ptx::tc_fence_after();
            const uint32_t q = warp & 3u, ch = warp >> 2;
            const uint32_t grow_e = row0 + q * 32u + lane;
            const float s2 = (KIND == K_NVFP4) ? __ldg((const float *)P.aux + e) : 1.f;
            const uint32_t c_begin = ch * (BN / 2), c_end = tmin<uint32_t>(c_begin + BN / 2, nt);
            for (uint32_t c0 = c_begin; c0 < c_end; c0 += 16) {
                uint32_t v[16];
                ptx::tmem_ld16(tmem + ((q * 32u) << 16) + c0, v);
                ptx::tmem_wait_ld();
                if (grow_e < P.n) {
#pragma unroll
                    for (int i = 0; i < 16; i++) {
                        const uint32_t col = c0 + i;
                        if (col < c_end)
                            store_out(P.out, P.out_dtype, (size_t)pairs_s[col] * P.n + grow_e,
                                      __uint_as_float(v[i]) * s2);
                    }
                }
            }
        }
        ptx::tc_fence_before();
    } else if (lane == 0) {
        // --------------------------------------------------------------- MMA issue
        const uint32_t idesc = ptx::idesc_f16(F16 ? 0u : 1u, nt_pad);
        uint32_t accum = 0;
        bool ok = true;
        for (uint32_t kt = 0; kt < P.ktiles; kt++) {
            const uint32_t s = kt % S, use = kt / S;
            if (!ptx::mbar_wait_bounded(full0 + 8 * s, use & 1u, abort_flag, P.err, ERR_TIMEOUT,
                                        P.timeout_ns)) {
                ok = false;
                break;
            }
            ptx::tc_fence_after();
            const uint32_t st = base + s * STAGE;
            const uint32_t a_hi = st, a_lo = st + A_TILE;
            const uint32_t b_hi = st + AT * A_TILE, b_lo = b_hi + B_TILE;
#pragma unroll
            for (int ks = 0; ks < KT / 16; ks++) {
                const uint32_t ko = ks * 32u;
                ptx::mma_f16_ss(tmem, ptx::sdesc_k128(a_hi + ko), ptx::sdesc_k128(b_hi + ko), idesc, accum);
                accum = 1;
                if constexpr (BT == 2)
                    ptx::mma_f16_ss(tmem, ptx::sdesc_k128(a_hi + ko), ptx::sdesc_k128(b_lo + ko), idesc, 1);
                if constexpr (AT == 2)
                    ptx::mma_f16_ss(tmem, ptx::sdesc_k128(a_lo + ko), ptx::sdesc_k128(b_hi + ko), idesc, 1);
            }
            ptx::mma_commit(empty0 + 8 * s);
        }
        ptx::mma_commit(accb);
        if (!ok) {
            // drain: the commit above tracks every MMA issued so far
            ptx::mbar_wait_bounded(accb, 0, nullptr, P.err, ERR_TIMEOUT, P.timeout_ns);
        }
    }
    __syncthreads();
    if (warp == MMA_WARP) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, BN);
    }
}

template <int KIND, int XT, int BN>
cudaError_t launch_t(const GemmParams &P0, uint32_t n_mtiles, uint32_t max_tiles, cudaStream_t st) {
    constexpr int AT = a_terms<KIND>();
    constexpr int BT = (XT == DT_F32) ? 2 : 1;
    constexpr int STAGE = AT * A_TILE + BT * BN * KT * 2;
    const int budget = BN >= 256 ? 200 * 1024 : 96 * 1024;
    int S = budget / STAGE;
    S = S < 2 ? 2 : (S > 6 ? 6 : S);
    GemmParams P = P0;
    P.stages = (uint32_t)S;
    const size_t smem = (size_t)S * STAGE + 1024;
    auto kern = grouped_gemm_kernel<KIND, XT, BN>;
    static int smem_set[64];
    cudaError_t e = ensure_dyn_smem(kern, smem, smem_set);
    if (e != cudaSuccess) return e;
    dim3 grid(n_mtiles, max_tiles);
    kern<<<grid, GEMM_THREADS, smem, st>>>(P);
    return cudaGetLastError();
}

template <int KIND, int BN>
cudaError_t launch_x(const GemmParams &P, int x_dtype, uint32_t nm, uint32_t mt, cudaStream_t st) {
    switch (x_dtype) {
        case DT_F32: return launch_t<KIND, DT_F32, BN>(P, nm, mt, st);
        case DT_BF16: return launch_t<KIND, DT_BF16, BN>(P, nm, mt, st);
        default: return launch_t<KIND, DT_F16, BN>(P, nm, mt, st);
    }
}

template <int BN>
cudaError_t launch_bn(const GemmParams &P, int kind, int x_dtype, uint32_t nm, uint32_t mt,
                      cudaStream_t st) {
    switch (kind) {
        case K_AFF4: return launch_x<K_AFF4, BN>(P, x_dtype, nm, mt, st);
        case K_AFF6: return launch_x<K_AFF6, BN>(P, x_dtype, nm, mt, st);
        case K_AFF8: return launch_x<K_AFF8, BN>(P, x_dtype, nm, mt, st);
        case K_CB2: return launch_x<K_CB2, BN>(P, x_dtype, nm, mt, st);
        case K_CB3: return launch_x<K_CB3, BN>(P, x_dtype, nm, mt, st);
        case K_CB4: return launch_x<K_CB4, BN>(P, x_dtype, nm, mt, st);
        case K_NVFP4: return launch_x<K_NVFP4, BN>(P, x_dtype, nm, mt, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

bool gemm_supported(const QmmArgs &a) {
    const uint32_t gs = a.group_size;
    if (gs < 16 || (gs & (gs - 1)) != 0) return false;
    if (a.k % 8 != 0 || a.k % gs != 0) return false;
    // packed codes are read with 8-byte loads (4-byte word loads for 3-bit codebook rows)
    if (a.row_bytes % (a.kind == K_CB3 ? 4u : 8u) != 0) return false;
    if ((uintptr_t)a.packed % 16 != 0 || (uintptr_t)a.x % 16 != 0) return false;
    if (a.num_experts > ROUTE_MAX_E) return false;
    return true;
}

uint32_t gemm_tile_rows(const QmmArgs &a) {
    const uint64_t R = (uint64_t)a.m * a.n_expert_used;
    return (R >= 96ull * a.num_experts) ? 256u : 64u;
}

cudaError_t launch_gemm(const QmmArgs &a, const uint32_t *offsets, const uint32_t *sorted_pairs,
                        const uint32_t *tiles, const uint32_t *tile_count, uint32_t max_tiles,
                        uint32_t *err, cudaStream_t st) {
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
    P.out_dtype = a.out_dtype;
    P.timeout_ns = WAIT_NS;
    const uint32_t nm = (a.n + BM - 1) / BM;
    if (gemm_tile_rows(a) == 256u) return launch_bn<256>(P, a.kind, a.x_dtype, nm, max_tiles, st);
    return launch_bn<64>(P, a.kind, a.x_dtype, nm, max_tiles, st);
}

}  // namespace moe
