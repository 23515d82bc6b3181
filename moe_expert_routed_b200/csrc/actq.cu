// actq.cu -- W4A4 activations: per-token NVFP4 quantisation of x.
//
// The pages quantise weights to NVFP4 (E2M1 codes, one E4M3 scale per 16
// values, a second-level f32 scale; spark_model helpers_a.rs) and name a grouped
// NVFP4 GEMM whose activations are NVFP4 too (metrale helpers_b.rs,
// build_cutlass_grouped_sfb), without saying how activations are quantised. The
// reading taken, per token t (one row of x), every step in f32:
//   g   = max_j |x[t][j]| / 2688   (2688 = 448 * 6: largest E4M3 scale times the
//                                   largest E2M1 value)
//   s_b = E4M3(max over block b of |x| / (6 g)), per block of 16 values, nearest
//         with ties to even, saturating at 448 (0 when g = 0)
//   q_j = E2M1(x[t][j] / (e4m3(s_b) g)), nearest with ties to even, saturating at
//         6, the quotient's sign kept (code 0 when the divisor is 0)
//   x^  = e2m1(q_j) * e4m3(s_b) * g
// The conversions are the hardware's round-to-nearest-even, satfinite ones.
//
// One CTA per token: a block-wide maximum, then two lanes per 16-value block.
#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr int AQ_THREADS = 256;

// E4M3 byte of v >= 0: round to nearest even, values above 448 to 448.
__device__ __forceinline__ uint32_t e4m3_rn_sat(float v) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(v));
    return r & 0xFFu;  // the second source lands in the low byte
}

__device__ __forceinline__ float e4m3_value(uint32_t b) {
    uint32_t h2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"((uint16_t)b));
    return __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu)));
}

// Two E2M1 codes in one byte: lo in bits 0-3, hi in bits 4-7.
__device__ __forceinline__ uint32_t e2m1x2_rn_sat(float lo, float hi) {
    uint32_t r;
    asm("{\n\t.reg .b8 t;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\t"
        "cvt.u32.u8 %0, t;\n\t}"
        : "=r"(r)
        : "f"(hi), "f"(lo));
    return r;
}

// Eight consecutive values of x from element i (i a multiple of 8): vector loads
// when the row is 16-byte aligned, else one at a time.
__device__ __forceinline__ void load8(const void *x, int dt, size_t i, bool vec, float (&v)[8]) {
    if (vec && dt == DT_F32) {
        const float4 a = __ldg((const float4 *)x + i / 4), b = __ldg((const float4 *)x + i / 4 + 1);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    } else if (vec) {
        const uint4 q = __ldg((const uint4 *)x + i / 8);
        const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int j = 0; j < 4; j++) {
            v[2 * j] = dt == DT_BF16 ? bf16_bits_to_f32(w[j] & 0xFFFFu) : f16_bits_to_f32(w[j] & 0xFFFFu);
            v[2 * j + 1] = dt == DT_BF16 ? bf16_bits_to_f32(w[j] >> 16) : f16_bits_to_f32(w[j] >> 16);
        }
    } else {
#pragma unroll
        for (int j = 0; j < 8; j++) v[j] = load_x(x, dt, i + j);
    }
}

// One CTA per token. Pass 1: the row's maximum. Pass 2: lanes 2p and 2p+1 of a warp
// take the two halves of one 16-value block (8 values each), so loads and stores
// are contiguous across the warp; every thread runs the same number of passes so
// that the pairs' shuffles always have both lanes.
__global__ void __launch_bounds__(AQ_THREADS)
quant_act_nvfp4(const void *__restrict__ x, int x_dtype, uint32_t k, uint8_t *__restrict__ codes,
                uint8_t *__restrict__ scales, float *__restrict__ gscale, float *__restrict__ xhat,
                uint16_t *__restrict__ x16) {
    __shared__ float red[AQ_THREADS / 32];
    const uint32_t t = blockIdx.x, tid = threadIdx.x, lane = tid & 31u;
    const size_t row = (size_t)t * k;
    const uint32_t k8 = k / 8u;  // 8-value chunks (even: k is a multiple of 16)
    const bool vec = ((uintptr_t)x & 15u) == 0;
    float a = 0.f;
    for (uint32_t c = tid; c < k8; c += AQ_THREADS) {
        float v[8];
        load8(x, x_dtype, row + 8u * c, vec, v);
#pragma unroll
        for (int j = 0; j < 8; j++) a = fmaxf(a, fabsf(v[j]));
    }
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, d));
    if (lane == 0) red[tid >> 5] = a;
    __syncthreads();
    a = red[0];
#pragma unroll
    for (int w = 1; w < AQ_THREADS / 32; w++) a = fmaxf(a, red[w]);
    const float g = __fdiv_rn(a, 2688.0f);
    if (tid == 0 && gscale) gscale[t] = g;
    const float six_g = __fmul_rn(6.0f, g);
    for (uint32_t c0 = 0; c0 < k8; c0 += AQ_THREADS) {
        const uint32_t c = c0 + tid;
        const bool valid = c < k8;
        float v[8], ab = 0.f;
        if (valid) {
            load8(x, x_dtype, row + 8u * c, vec, v);
        } else {
#pragma unroll
            for (int j = 0; j < 8; j++) v[j] = 0.f;
        }
#pragma unroll
        for (int j = 0; j < 8; j++) ab = fmaxf(ab, fabsf(v[j]));
        ab = fmaxf(ab, __shfl_xor_sync(0xFFFFFFFFu, ab, 1));  // the block's other half
        if (!valid) continue;
        const uint32_t s = g > 0.f ? e4m3_rn_sat(__fdiv_rn(ab, six_g)) : 0u;
        if (scales && (c & 1u) == 0) scales[row / 16u + c / 2u] = (uint8_t)s;
        const float sv = e4m3_value(s);
        const float d = __fmul_rn(sv, g);
        uint32_t cw = 0;
        float vs[8];
#pragma unroll
        for (int j = 0; j < 8; j += 2) {
            const uint32_t c2 = d > 0.f ? e2m1x2_rn_sat(__fdiv_rn(v[j], d), __fdiv_rn(v[j + 1], d)) : 0u;
            cw |= c2 << (4 * j);
            vs[j] = e2m1_to_f32(c2 & 15u) * sv;  // exact: at most 6 significant bits
            vs[j + 1] = e2m1_to_f32(c2 >> 4) * sv;
        }
        if (codes) *(uint32_t *)(codes + (row + 8u * c) / 2) = cw;
        if (xhat) {
            float4 *o = (float4 *)(xhat + row + 8u * c);
            o[0] = make_float4(__fmul_rn(vs[0], g), __fmul_rn(vs[1], g), __fmul_rn(vs[2], g), __fmul_rn(vs[3], g));
            o[1] = make_float4(__fmul_rn(vs[4], g), __fmul_rn(vs[5], g), __fmul_rn(vs[6], g), __fmul_rn(vs[7], g));
        }
        if (x16) {
            uint32_t h[4];
#pragma unroll
            for (int j = 0; j < 4; j++)
                h[j] = (__float_as_uint(vs[2 * j]) >> 16) | (__float_as_uint(vs[2 * j + 1]) & 0xFFFF0000u);
            *(uint4 *)(x16 + row + 8u * c) = make_uint4(h[0], h[1], h[2], h[3]);
        }
    }
}

}  // namespace

cudaError_t launch_quant_act(const void *x, int x_dtype, uint32_t m, uint32_t k, uint8_t *codes, uint8_t *scales,
                             float *gscale, float *xhat, uint16_t *x16, cudaStream_t st) {
    if (m == 0) return cudaSuccess;
    if (k == 0 || k % 16u != 0 || ((uintptr_t)codes & 3u) || ((uintptr_t)xhat & 15u) || ((uintptr_t)x16 & 15u))
        return cudaErrorInvalidValue;
    quant_act_nvfp4<<<m, AQ_THREADS, 0, st>>>(x, x_dtype, k, codes, scales, gscale, xhat, x16);
    return cudaGetLastError();
}

}  // namespace moe
