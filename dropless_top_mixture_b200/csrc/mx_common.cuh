// MXFP8 block codec on the device: one block = 32 consecutive values of a
// row sharing one scale ("olmoforge" README, "MXFP8 分块量化"; E4M3 payload).
//   s = fp32(amax / 448) (1 for an all-zero block); UE8M0 mode rounds s up to
//   the next power of two with the exponent clamped to [-127, 127];
//   q = E4M3(fp32(v / s)), round-to-nearest-even, saturating to ±448.
#pragma once

#include <cuda_fp8.h>

#include "common.cuh"

namespace moe {
namespace mxc {

// Smallest e with 2^e >= s for a positive finite fp32 s, clamped to
// [-127, 127]. Works from the bit pattern so no rounding is involved.
__device__ __forceinline__ int pow2_ceil_exp(float s) {
    const uint32_t u = __float_as_uint(s);
    const int be = (int)((u >> 23) & 0xFF);
    const uint32_t man = u & 0x7FFFFFu;
    int e;
    if (be == 0) {
        // subnormal: s = man * 2^-149, man in [1, 2^23)
        const int msb = 31 - __clz((int)man);
        e = msb - 149 + ((man & (man - 1)) ? 1 : 0);
    } else {
        e = be - 127 + (man ? 1 : 0);
    }
    return e < -127 ? -127 : (e > 127 ? 127 : e);
}

// 2^e for e in [-127, 127] as an fp32 bit pattern (2^-127 is subnormal)
__device__ __forceinline__ float exp2_exact(int e) {
    return e >= -126 ? __uint_as_float((uint32_t)(e + 127) << 23) : __uint_as_float(0x00400000u);
}

// UE8M0 block scale of 32 values: returns the biased exponent byte and the
// scale value.
__device__ __forceinline__ uint8_t e8m0_scale(const float* v, float* scale) {
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
    const int e = (amax == 0.f) ? 0 : pow2_ceil_exp(__fdiv_rn(amax, 448.0f));
    *scale = exp2_exact(e);
    return (uint8_t)(e + 127);
}

// 32 values / 2^(sbyte - 127) -> 32 E4M3 codes packed in 8 words. The
// division by a power of two is a multiplication by its exact reciprocal
// 2^(127 - sbyte), which is rounded once to the same fp32 value.
__device__ __forceinline__ void encode32_e8m0(const float* v, uint8_t sbyte, uint32_t* w) {
    const float inv = exp2_exact(127 - (int)sbyte);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        uint32_t word = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const __nv_fp8_storage_t c =
                __nv_cvt_float_to_fp8(v[4 * i + j] * inv, __NV_SATFINITE, __NV_E4M3);
            word |= (uint32_t)c << (8 * j);
        }
        w[i] = word;
    }
}

// 32 values / scale -> 32 E4M3 codes packed in 8 words.
__device__ __forceinline__ void encode32(const float* v, float scale, uint32_t* w) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        uint32_t word = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const __nv_fp8_storage_t c =
                __nv_cvt_float_to_fp8(__fdiv_rn(v[4 * i + j], scale), __NV_SATFINITE, __NV_E4M3);
            word |= (uint32_t)c << (8 * j);
        }
        w[i] = word;
    }
}

}  // namespace mxc
}  // namespace moe
