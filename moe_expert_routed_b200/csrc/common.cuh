// common.cuh -- shared device helpers of the CUDA path: number formats, storage
// constants, error word bits. Independent of the CPU oracle.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

enum Fmt : int { FMT_AFFINE = 0, FMT_CODEBOOK = 1, FMT_NVFP4 = 2, FMT_MXFP4 = 3 };
enum DType : int { DT_F32 = 0, DT_BF16 = 1, DT_F16 = 2 };

// Storage kinds: one per (format, bits) pair the kernels are specialised for.
enum Kind : int { K_AFF4 = 0, K_AFF6, K_AFF8, K_CB2, K_CB3, K_CB4, K_NVFP4, K_MXFP4, K_COUNT };

// Device error word bits (first u32 of the workspace).
constexpr uint32_t ERR_BAD_ID = 1u;
constexpr uint32_t ERR_TIMEOUT = 2u;
constexpr uint32_t ERR_INTERNAL = 4u;
constexpr uint32_t ERR_BAD_POINTER = 8u;  // pointer-table weights: missing or misaligned scales / biases

__host__ __device__ inline int kind_of(int fmt, int bits) {
    if (fmt == FMT_AFFINE) return bits == 4 ? K_AFF4 : bits == 6 ? K_AFF6 : bits == 8 ? K_AFF8 : -1;
    if (fmt == FMT_CODEBOOK) return bits == 2 ? K_CB2 : bits == 3 ? K_CB3 : bits == 4 ? K_CB4 : -1;
    if (fmt == FMT_NVFP4) return bits == 4 ? K_NVFP4 : -1;
    if (fmt == FMT_MXFP4) return bits == 4 ? K_MXFP4 : -1;
    return -1;
}

// Bits per code of each kind.
__host__ __device__ constexpr int kind_bits(int kind) {
    return kind == K_AFF4 ? 4 : kind == K_AFF6 ? 6 : kind == K_AFF8 ? 8 : kind == K_CB2 ? 2
         : kind == K_CB3 ? 3 : 4;
}

template <typename T>
__host__ __device__ __forceinline__ T tmin(T a, T b) { return a < b ? a : b; }

// --------------------------------------------------------------- decoders

// bf16 -> f32: the bf16 pattern is the high half of the f32 pattern.
__device__ __forceinline__ float bf16_bits_to_f32(uint32_t h) { return __uint_as_float(h << 16); }

__device__ __forceinline__ float f16_bits_to_f32(uint32_t h) {
    return __half2float(__ushort_as_half((unsigned short)h));
}

// OCP FP8 E4M3 (FN): bias 7, exponent field 0 = subnormal m * 2^-9, 0x7F/0xFF NaN.
__device__ __forceinline__ float e4m3_to_f32(uint32_t b) {
    uint32_t s = (b >> 7) & 1u, e = (b >> 3) & 15u, m = b & 7u;
    float mag = (e == 0u) ? (float)m * 0.001953125f                       // m * 2^-9
                          : __uint_as_float(((e + 120u) << 23) | (m << 20)); // (1+m/8)*2^(e-7)
    if (e == 15u && m == 7u) mag = __uint_as_float(0x7FC00000u);
    return s ? -mag : mag;
}

// OCP MX FP4 E2M1: bias 1, exponent field 0 = subnormal m * 0.5, no NaN/Inf.
// OCP Microscaling E8M0 scale byte: 2^(b - 127); 0xFF is NaN, 0 the subnormal 2^-127.
__device__ __forceinline__ float e8m0_to_f32(uint32_t b) {
    if (b == 0xFFu) return __uint_as_float(0x7FC00000u);
    return b ? __uint_as_float(b << 23) : __uint_as_float(0x00400000u);
}

__device__ __forceinline__ float e2m1_to_f32(uint32_t c) {
    uint32_t s = (c >> 3) & 1u, e = (c >> 1) & 3u, m = c & 1u;
    float mag = (e == 0u) ? 0.5f * (float)m : __uint_as_float(((e + 126u) << 23) | (m << 22));
    return s ? -mag : mag;
}

__device__ __forceinline__ float load_x(const void *x, int dt, size_t idx) {
    if (dt == DT_F32) return __ldg((const float *)x + idx);
    uint32_t h = __ldg((const unsigned short *)x + idx);
    return dt == DT_BF16 ? bf16_bits_to_f32(h) : f16_bits_to_f32(h);
}

// Per-expert output bias (f32, bf16 or f16) at element idx of [num_experts, n];
// 0 without a bias.
__device__ __forceinline__ float load_bias(const void *bias, int dt, size_t idx) {
    if (!bias) return 0.f;
    return load_x(bias, dt, idx);
}

__device__ __forceinline__ void store_out(void *out, int dt, size_t idx, float v) {
    if (dt == DT_F32) {
        ((float *)out)[idx] = v;
    } else if (dt == DT_BF16) {
        ((__nv_bfloat16 *)out)[idx] = __float2bfloat16_rn(v);
    } else {
        ((__half *)out)[idx] = __float2half_rn(v);
    }
}

// ------------------------------------------------ gated (GLU) output epilogue
//
// The fused gate+up projection (spark_model helpers_a.rs, MoeLayer: the fused
// gate+up kernel with SiLU, or GELU for GeGLU experts via set_gelu_activation):
// with n weight rows per expert, rows [0, n/2) are the gate and rows [n/2, n)
// the up projection, and the output element j of a pair is act(gate_j) * up_j.
// The kernels walk "logical" rows in which gate and up rows alternate, so that
// both halves of an output land next to each other: logical row L is weight row
// L/2 (L even, gate) or n/2 + L/2 (L odd, up). nh = n/2, or 0 without GLU.
__host__ __device__ __forceinline__ uint32_t glu_row(uint32_t L, uint32_t nh) {
    return nh ? ((L & 1u) ? nh + (L >> 1) : (L >> 1)) : L;
}

// act(g) in fp32: 0 SiLU g / (1 + e^-g); 1 GELU, tanh form
// g/2 (1 + tanh(sqrt(2/pi) (g + 0.044715 g^3))); 2 GELU, erf form g/2 (1 + erf(g / sqrt 2)).
__device__ __forceinline__ float glu_act(int act, float g) {
    if (act == 0) return g / (1.f + expf(-g));
    if (act == 1) return 0.5f * g * (1.f + tanhf(0.7978845608f * fmaf(0.044715f * g * g, g, g)));
    return 0.5f * g * (1.f + erff(g * 0.70710678f));
}

}  // namespace moe
