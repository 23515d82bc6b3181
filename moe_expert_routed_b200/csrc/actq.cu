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
// One CTA per token: a block-wide maximum, then one thread per 16-value block.
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

__global__ void __launch_bounds__(AQ_THREADS)
quant_act_nvfp4(const void *__restrict__ x, int x_dtype, uint32_t k, uint8_t *__restrict__ codes,
                uint8_t *__restrict__ scales, float *__restrict__ gscale, float *__restrict__ xhat) {
    __shared__ float red[AQ_THREADS / 32];
    const uint32_t t = blockIdx.x, tid = threadIdx.x;
    const size_t row = (size_t)t * k;
    float a = 0.f;
    for (uint32_t j = tid; j < k; j += AQ_THREADS) a = fmaxf(a, fabsf(load_x(x, x_dtype, row + j)));
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, d));
    if ((tid & 31u) == 0) red[tid >> 5] = a;
    __syncthreads();
    a = red[0];
#pragma unroll
    for (int w = 1; w < AQ_THREADS / 32; w++) a = fmaxf(a, red[w]);
    const float g = __fdiv_rn(a, 2688.0f);
    if (tid == 0 && gscale) gscale[t] = g;
    const float six_g = __fmul_rn(6.0f, g);
    for (uint32_t b = tid; b < k / 16u; b += AQ_THREADS) {
        float v[16], ab = 0.f;
#pragma unroll
        for (int i = 0; i < 16; i++) {
            v[i] = load_x(x, x_dtype, row + 16u * b + i);
            ab = fmaxf(ab, fabsf(v[i]));
        }
        const uint32_t s = g > 0.f ? e4m3_rn_sat(__fdiv_rn(ab, six_g)) : 0u;
        if (scales) scales[(size_t)t * (k / 16u) + b] = (uint8_t)s;
        const float sv = e4m3_value(s);
        const float d = __fmul_rn(sv, g);
        uint32_t packed[2] = {0u, 0u};
#pragma unroll
        for (int i = 0; i < 16; i += 2) {
            const uint32_t c2 = d > 0.f ? e2m1x2_rn_sat(__fdiv_rn(v[i], d), __fdiv_rn(v[i + 1], d)) : 0u;
            packed[i / 8] |= c2 << (8 * ((i % 8) / 2));
            if (xhat) {
                xhat[row + 16u * b + i] = __fmul_rn(__fmul_rn(e2m1_to_f32(c2 & 15u), sv), g);
                xhat[row + 16u * b + i + 1] = __fmul_rn(__fmul_rn(e2m1_to_f32(c2 >> 4), sv), g);
            }
        }
        if (codes) *(uint2 *)(codes + (row + 16u * b) / 2) = make_uint2(packed[0], packed[1]);
    }
}

}  // namespace

cudaError_t launch_quant_act(const void *x, int x_dtype, uint32_t m, uint32_t k, uint8_t *codes, uint8_t *scales,
                             float *gscale, float *xhat, cudaStream_t st) {
    if (m == 0) return cudaSuccess;
    if (k == 0 || k % 16u != 0 || ((uintptr_t)codes & 7u)) return cudaErrorInvalidValue;
    quant_act_nvfp4<<<m, AQ_THREADS, 0, st>>>(x, x_dtype, k, codes, scales, gscale, xhat);
    return cudaGetLastError();
}

}  // namespace moe
