// MXFP8 block quantisation of the MoE layer's operands.
//
// "olmoforge" README, "MXFP8 分块量化": blocks of 32 values share one scale
// derived from the block's largest magnitude and the E4M3 maximum (448);
// the Olmo-core 3 news article (xxqk.cn), "三招拆分、三项优化、一个精度开关",
// names MXFP8 as the low-precision switch. The payload is E4M3 (OCP FP8):
// q = E4M3_rne_satfinite(fp32(v / s)), s = fp32(amax / 448) (1 when the block
// is all zero), optionally rounded up to a power of two (UE8M0, the scale
// format block-scaled MMA consumes).
//
// One thread per 32-element block: it reads the block (64 or 128 bytes),
// finds amax, derives the scale and writes 32 code bytes plus one scale.
#include "mx_common.cuh"

namespace moe {
namespace mx {

constexpr int THREADS = 256;

using mxc::exp2_exact;
using mxc::pow2_ceil_exp;

template <int DT>
__device__ __forceinline__ void load32(const void* in, int64_t blk, float* v) {
    if (DT == MOE_BF16) {
        const uint4* p = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(in) + blk * 32);
#pragma unroll
        for (int i = 0; i < 4; ++i) unpack8(__ldcs(p + i), v + 8 * i);
    } else {
        const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(in) + blk * 32);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float4 f = __ldcs(p + i);
            v[4 * i] = f.x; v[4 * i + 1] = f.y; v[4 * i + 2] = f.z; v[4 * i + 3] = f.w;
        }
    }
}

template <int DT, int MODE>
__global__ void __launch_bounds__(THREADS) quantize_kernel(const void* __restrict__ in,
                                                           int64_t nblocks,
                                                           uint8_t* __restrict__ q,
                                                           void* __restrict__ scales) {
    for (int64_t b = (int64_t)blockIdx.x * THREADS + threadIdx.x; b < nblocks;
         b += (int64_t)gridDim.x * THREADS) {
        float v[32];
        load32<DT>(in, b, v);
        float amax = 0.f;
#pragma unroll
        for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
        const float s32 = __fdiv_rn(amax, 448.0f);
        float s, inv = 1.f;
        if (MODE == MOE_SCALE_F32) {
            s = (amax == 0.f) ? 1.0f : s32;
            static_cast<float*>(scales)[b] = s;
        } else {
            const int e = (amax == 0.f) ? 0 : pow2_ceil_exp(s32);
            s = exp2_exact(e);
            inv = exp2_exact(-e);
            static_cast<uint8_t*>(scales)[b] = (uint8_t)(e + 127);
        }
        uint32_t w[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            uint32_t word = 0;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                // a UE8M0 scale is a power of two: divide by multiplying by its
                // exact reciprocal (the same rounded value)
                const float qv = MODE == MOE_SCALE_E8M0 ? v[4 * i + j] * inv : __fdiv_rn(v[4 * i + j], s);
                const __nv_fp8_storage_t c = __nv_cvt_float_to_fp8(qv, __NV_SATFINITE, __NV_E4M3);
                word |= (uint32_t)c << (8 * j);
            }
            w[i] = word;
        }
        uint4* dst = reinterpret_cast<uint4*>(q + b * 32);
        dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
        dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
    }
}

template <int MODE>
__global__ void __launch_bounds__(THREADS) dequantize_kernel(const uint8_t* __restrict__ q,
                                                             const void* __restrict__ scales,
                                                             int64_t nblocks,
                                                             __nv_bfloat16* __restrict__ out) {
    for (int64_t b = (int64_t)blockIdx.x * THREADS + threadIdx.x; b < nblocks;
         b += (int64_t)gridDim.x * THREADS) {
        const float s = (MODE == MOE_SCALE_F32)
                            ? static_cast<const float*>(scales)[b]
                            : exp2_exact((int)static_cast<const uint8_t*>(scales)[b] - 127);
        const uint4* src = reinterpret_cast<const uint4*>(q + b * 32);
        uint4* dst = reinterpret_cast<uint4*>(out + b * 32);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const uint4 c = src[h];
            const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
            float f[16];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const __half_raw hr = __nv_cvt_fp8_to_halfraw(
                        (__nv_fp8_storage_t)((cw[i] >> (8 * j)) & 0xFF), __NV_E4M3);
                    f[4 * i + j] = __half2float(__half(hr)) * s;
                }
            dst[2 * h] = pack8(f);
            dst[2 * h + 1] = pack8(f + 8);
        }
    }
}

inline int grid_for(int64_t nblocks) {
    int64_t g = (nblocks + THREADS - 1) / THREADS;
    const int64_t cap = (int64_t)num_sms() * 16;
    return (int)(g < cap ? g : cap);
}

}  // namespace mx
}  // namespace moe

using namespace moe;

extern "C" int mxfp8_quantize(const void* in, int dtype, int64_t rows, int64_t cols,
                              int scale_mode, uint8_t* q, void* scales, void* stream) {
    if (rows < 0 || cols <= 0 || cols % 32 != 0) return MOE_ERR_INVALID;
    if (dtype != MOE_BF16 && dtype != MOE_F32) return MOE_ERR_UNSUPPORTED;
    if (scale_mode != MOE_SCALE_F32 && scale_mode != MOE_SCALE_E8M0) return MOE_ERR_INVALID;
    if (rows == 0) return MOE_OK;
    if (!in || !q || !scales || !aligned16(in) || !aligned16(q)) return MOE_ERR_INVALID;
    if (check_only()) return MOE_OK;
    const int64_t nb = rows * (cols / 32);
    cudaStream_t st = as_stream(stream);
    const int g = mx::grid_for(nb);
    if (dtype == MOE_BF16) {
        if (scale_mode == MOE_SCALE_F32)
            mx::quantize_kernel<MOE_BF16, MOE_SCALE_F32><<<g, mx::THREADS, 0, st>>>(in, nb, q, scales);
        else
            mx::quantize_kernel<MOE_BF16, MOE_SCALE_E8M0><<<g, mx::THREADS, 0, st>>>(in, nb, q, scales);
    } else {
        if (scale_mode == MOE_SCALE_F32)
            mx::quantize_kernel<MOE_F32, MOE_SCALE_F32><<<g, mx::THREADS, 0, st>>>(in, nb, q, scales);
        else
            mx::quantize_kernel<MOE_F32, MOE_SCALE_E8M0><<<g, mx::THREADS, 0, st>>>(in, nb, q, scales);
    }
    return launch_status();
}

extern "C" int mxfp8_dequantize(const uint8_t* q, const void* scales, int scale_mode,
                                int64_t rows, int64_t cols, void* out_bf16, void* stream) {
    if (rows < 0 || cols <= 0 || cols % 32 != 0) return MOE_ERR_INVALID;
    if (scale_mode != MOE_SCALE_F32 && scale_mode != MOE_SCALE_E8M0) return MOE_ERR_INVALID;
    if (rows == 0) return MOE_OK;
    if (!q || !scales || !out_bf16 || !aligned16(q) || !aligned16(out_bf16)) return MOE_ERR_INVALID;
    if (check_only()) return MOE_OK;
    const int64_t nb = rows * (cols / 32);
    cudaStream_t st = as_stream(stream);
    const int g = mx::grid_for(nb);
    __nv_bfloat16* o = static_cast<__nv_bfloat16*>(out_bf16);
    if (scale_mode == MOE_SCALE_F32)
        mx::dequantize_kernel<MOE_SCALE_F32><<<g, mx::THREADS, 0, st>>>(q, scales, nb, o);
    else
        mx::dequantize_kernel<MOE_SCALE_E8M0><<<g, mx::THREADS, 0, st>>>(q, scales, nb, o);
    return launch_status();
}
