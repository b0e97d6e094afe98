// common.cuh -- device helpers shared by the CSA/HCA kernels (sm_100a).
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <stdint.h>

namespace csa {

enum Dtype : int { DT_F32 = 0, DT_BF16 = 1, DT_E4M3 = 2, DT_E4M3H = 3 };

// Order-preserving map of an fp32 score to an unsigned radix key: a larger
// score gives a larger key, negative scores sort below every zero, and -0
// and +0 share one key (they are equal scores).
__device__ __forceinline__ uint32_t score_key(float x) {
    const uint32_t u = __float_as_uint(x);
    return x == 0.0f ? 0x80000000u : (u ^ ((uint32_t)((int32_t)u >> 31) | 0x80000000u));
}

// Normalised Walsh-Hadamard rotation of a row of d fp32 values (d a power of
// two) in shared memory, by one warp, in the order the fp8 Hadamard type
// defines: for stride s = 1, 2, ..., d/2 every pair (i, i+s) with i & s == 0
// becomes (x_i + x_{i+s}, x_i - x_{i+s}); then each value is multiplied by
// norm = fp32(1/sqrt(d)) (computed on the host, passed in).
__device__ __forceinline__ void hadamard_row_warp(float* row, int d, float norm) {
    const int lane = threadIdx.x & 31;
    for (int s = 1; s < d; s <<= 1) {
        for (int p = lane; p < d / 2; p += 32) {
            const int i = (p / s) * 2 * s + (p % s);
            const float a = row[i], b = row[i + s];
            row[i] = a + b;
            row[i + s] = a - b;
        }
        __syncwarp();
    }
    for (int i = lane; i < d; i += 32) row[i] = row[i] * norm;
    __syncwarp();
}

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

__device__ __forceinline__ float e4m3_value(uint8_t code) {
    __nv_fp8_e4m3 v;
    v.__x = code;
    return static_cast<float>(v);
}

// nearest-even, saturating to +-448 (the largest finite E4M3 magnitude)
__device__ __forceinline__ uint8_t e4m3_code(float x) {
    return static_cast<uint8_t>(__nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3));
}

template <typename T>
__device__ __forceinline__ void store_out(T* p, float v);
template <>
__device__ __forceinline__ void store_out<float>(float* p, float v) { *p = v; }
template <>
__device__ __forceinline__ void store_out<__nv_bfloat16>(__nv_bfloat16* p, float v) {
    *p = __float2bfloat16_rn(v);
}

// ReLU that maps -0 to +0, so a non-negative score's bit pattern orders like its value
__device__ __forceinline__ float relu0(float x) { return x > 0.0f ? x : 0.0f; }

__device__ __forceinline__ int clampi(int v, int lo, int hi) { return v < lo ? lo : (v > hi ? hi : v); }

}  // namespace csa
