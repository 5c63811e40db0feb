// common.cuh -- small device helpers shared by the kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace rq {

__device__ __forceinline__ float bf16_to_f32(uint16_t bits) { return __uint_as_float((uint32_t)bits << 16); }

// FP8 E4M3 byte -> float (exact; E4M3 is a subset of FP16).
__device__ __forceinline__ float e4m3_to_f32(uint32_t byte) {
    __half_raw hr = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)(byte & 0xFF), __NV_E4M3);
    return __half2float(__half(hr));
}

__device__ __forceinline__ double e4m3_to_f64(uint32_t byte) { return (double)e4m3_to_f32(byte); }

// Round a double to FP8 E4M3 (nearest, ties to even, saturating to +-448).
__device__ __forceinline__ uint32_t f64_to_e4m3(double v) {
    return (uint32_t)__nv_cvt_double_to_fp8(v, __NV_SATFINITE, __NV_E4M3);
}

// Sign bit j of the seeded diagonal sigma (1 -> multiply by -1).
__device__ __forceinline__ bool sigma_neg(const uint32_t sigma[4], int j) { return (sigma[j >> 5] >> (j & 31)) & 1u; }

// In-warp fast Walsh-Hadamard transform of a 128-vector held as 4
// consecutive elements per lane (element 4*lane + k in v[k]); computes
// H_128 v in Sylvester (natural) order, unnormalised.
template <typename T>
__device__ __forceinline__ void wht128_warp(T v[4], int lane) {
    T a0 = v[0] + v[1], a1 = v[0] - v[1], a2 = v[2] + v[3], a3 = v[2] - v[3];
    v[0] = a0 + a2;
    v[2] = a0 - a2;
    v[1] = a1 + a3;
    v[3] = a1 - a3;
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {
        const bool upper = (lane & m) != 0;
#pragma unroll
        for (int k = 0; k < 4; k++) {
            T other = __shfl_xor_sync(0xffffffffu, v[k], m);
            v[k] = upper ? (other - v[k]) : (v[k] + other);
        }
    }
}

// The transform of two 128-vectors at once (independent shuffle chains
// interleaved).
template <typename T>
__device__ __forceinline__ void wht128_warp2(T u[4], T v[4], int lane) {
    {
        T a0 = u[0] + u[1], a1 = u[0] - u[1], a2 = u[2] + u[3], a3 = u[2] - u[3];
        u[0] = a0 + a2;
        u[2] = a0 - a2;
        u[1] = a1 + a3;
        u[3] = a1 - a3;
        T b0 = v[0] + v[1], b1 = v[0] - v[1], b2 = v[2] + v[3], b3 = v[2] - v[3];
        v[0] = b0 + b2;
        v[2] = b0 - b2;
        v[1] = b1 + b3;
        v[3] = b1 - b3;
    }
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {
        const bool upper = (lane & m) != 0;
#pragma unroll
        for (int k = 0; k < 4; k++) {
            const T ou = __shfl_xor_sync(0xffffffffu, u[k], m);
            const T ov = __shfl_xor_sync(0xffffffffu, v[k], m);
            u[k] = upper ? (ou - u[k]) : (u[k] + ou);
            v[k] = upper ? (ov - v[k]) : (v[k] + ov);
        }
    }
}

}  // namespace rq
