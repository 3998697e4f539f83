// Backward of the MXFP8 expert FFN (sm_100a).
//
// "专家池 8→128 只慢 5%…" (xxqk.cn), section "三招拆分、三项优化、一个精度开关":
// the MXFP8 switch speeds up training, the gain coming from the feed-forward
// computation and the expert data movement; "olmoforge" README, capability
// table and "MXFP8 分块量化": 32-element blocks sharing one scale. The pages do
// not spell out the precision of the backward; the reading taken here:
//
//   the two input-gradient GEMMs run on block-scaled FP8 like the forward,
//   every operand quantised (UE8M0 scales, E4M3 codes) along its own
//   contraction dimension:
//     dH  = Q(dYe) · Q(W2_e)ᵀ-by-d        K = d: dYe along d, W2_e along d
//     dXe = Q([dA | dB]) · Q([W1_e; W3_e]) K = 2F: along F
//   the weight gradients stay bf16 tensor-core GEMMs (the bf16 weight
//   gradients of "OLMo-core 3 发布：主攻混合专家训练与导出校验", 主要功能) over the
//   forward's own dequantised operands: dW1 = dAᵀ·deq(Xq), dW3 = dBᵀ·deq(Xq),
//   dW2 = dYeᵀ·deq(Hq);
//   dYe = bf16(gate · dOut[t]) (the scaled dispatch of the bf16 backward);
//   dA = dH·B·silu'(A), dB = dH·silu(A) in fp32 from the bf16 dH and the
//   forward's saved bf16 pre-activations A, B, stored in bf16 for the weight
//   gradients and quantised from their fp32 values for dXe.
//
// The FP8 GEMMs are the forward's down kernel (moe_grouped_down_mxfp8) with
// the backward weights: W2 re-quantised along d as [E, F, d] and W1, W3
// re-quantised along F as one [E, d, 2F] tensor (mxfp8_quantize_weights_bwd,
// once per weight update, like the forward's weight quantisation).
#include "mx_common.cuh"

namespace moe {

// bf16 weight gradients of the grouped SwiGLU FFN (backward.cu)
int swiglu_wgrad(const void* Xe, const void* dA, const void* dB, const void* dYe, const void* H,
                 const int32_t* offsets, int64_t E, int64_t R, int64_t d, int64_t F, void* dW1,
                 void* dW3, void* dW2, cudaStream_t st);

namespace mxb {

constexpr int TQ_ROWS = 32;  // input rows per CTA = one scale block of the output
constexpr int TQ_COLS = 64;  // input columns per CTA = output rows

// Out[e][c][col_off + r] = E4M3 code of In[e][r][c], quantised along r in
// blocks of 32 (UE8M0 scale byte at S[e][c][(col_off + r) / 32]).
//   In [E][rows][cols] bf16, row stride cols, expert stride in_es elements;
//   Q [E][cols][ldq] uint8; S [E][cols][ldq / 32] uint8.
// One CTA stages 32 input rows x 64 input columns in shared memory (rows read
// as 128-byte segments); thread c then quantises output row c0 + c.
__global__ void __launch_bounds__(256)
    transpose_quant_kernel(const __nv_bfloat16* __restrict__ in, int64_t in_es, int rows, int cols,
                           uint8_t* __restrict__ q, uint8_t* __restrict__ s, int ldq, int col_off) {
    __shared__ float tile[TQ_ROWS][TQ_COLS + 1];
    const int e = blockIdx.z;
    const int r0 = blockIdx.y * TQ_ROWS, c0 = blockIdx.x * TQ_COLS;
    const __nv_bfloat16* src = in + (int64_t)e * in_es;
    for (int i = threadIdx.x; i < TQ_ROWS * TQ_COLS; i += blockDim.x) {
        const int rr = i / TQ_COLS, cc = i - rr * TQ_COLS;
        tile[rr][cc] = c0 + cc < cols ? __bfloat162float(src[(int64_t)(r0 + rr) * cols + c0 + cc])
                                      : 0.f;
    }
    __syncthreads();
    const int c = c0 + (int)threadIdx.x;
    if (threadIdx.x >= TQ_COLS || c >= cols || r0 >= rows) return;
    float v[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = tile[j][threadIdx.x];
    float sc;
    const uint8_t sb = mxc::e8m0_scale(v, &sc);
    uint32_t w[8];
    mxc::encode32_e8m0(v, sb, w);
    const int64_t orow = (int64_t)e * cols + c;
    uint4* dq = reinterpret_cast<uint4*>(q + orow * ldq + col_off + r0);
    dq[0] = make_uint4(w[0], w[1], w[2], w[3]);
    dq[1] = make_uint4(w[4], w[5], w[6], w[7]);
    s[orow * (ldq / 32) + (col_off + r0) / 32] = sb;
}

static int transpose_quant(const void* in, int64_t in_es, int64_t E, int64_t rows, int64_t cols,
                           uint8_t* q, uint8_t* s, int64_t ldq, int64_t col_off, cudaStream_t st) {
    const dim3 grid((unsigned)((cols + TQ_COLS - 1) / TQ_COLS), (unsigned)(rows / TQ_ROWS),
                    (unsigned)E);
    transpose_quant_kernel<<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(in), in_es,
                                                 (int)rows, (int)cols, q, s, (int)ldq,
                                                 (int)col_off);
    return launch_status();
}

__device__ __forceinline__ float sigmoid_(float a) { return 1.0f / (1.0f + __expf(-a)); }

// The pairwise SwiGLU backward dA = dH·B·silu'(A), dB = dH·silu(A)
// (silu'(a) = s(1 + a(1 - s)), s = sigmoid(a)) in fp32; dA, dB stored in
// bf16 [R, F]; the fp32 values quantised into Q [R, 2F] (dA in columns
// 0..F-1, dB in F..2F-1) with scale bytes S [R, 2F/32]. Four lanes share a
// 32-column block, eight columns each: a warp reads and writes 512
// contiguous bytes of a row per access, and the block's maximum is two
// shuffles among the four lanes. F % 32 == 0, so a block's lanes are
// consecutive lanes of one warp.
// 8 values / 2^e -> 8 E4M3 codes, dividing by the power of two as a
// multiplication by its exact reciprocal (the same rounded value)
__device__ __forceinline__ uint2 encode8(const float* v, int e) {
    const float inv = mxc::exp2_exact(-e);
    uint32_t w[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        uint32_t word = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const __nv_fp8_storage_t c =
                __nv_cvt_float_to_fp8(v[4 * i + j] * inv, __NV_SATFINITE, __NV_E4M3);
            word |= (uint32_t)c << (8 * j);
        }
        w[i] = word;
    }
    return make_uint2(w[0], w[1]);
}

// UE8M0 scale exponent of a block whose 32 values are spread over 4
// consecutive lanes (8 each); every lane of the four gets it.
__device__ __forceinline__ int e8m0_exp_4lanes(const float* v) {
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    return (amax == 0.f) ? 0 : mxc::pow2_ceil_exp(__fdiv_rn(amax, 448.0f));
}

__global__ void __launch_bounds__(256)
    swiglu_bwd_quant_kernel(const __nv_bfloat16* __restrict__ dH,
                            const __nv_bfloat16* __restrict__ A,
                            const __nv_bfloat16* __restrict__ B, int64_t R, int F,
                            __nv_bfloat16* __restrict__ dA, __nv_bfloat16* __restrict__ dB,
                            uint8_t* __restrict__ q, uint8_t* __restrict__ s) {
    const int per_row = F / 8;  // 8-column pieces per row (a multiple of 4)
    const int nb = F / 32;
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    // R * per_row is a multiple of 4, so the four lanes of a block are all
    // live or all past the end; the dead ones still take part in the shuffles
    const bool live = i < R * (int64_t)per_row;
    const int64_t r = live ? i / per_row : 0;
    const int c8 = live ? (int)(i - r * per_row) : 0;
    const int64_t off = r * F + 8 * (int64_t)c8;
    float da[8], db[8];
    if (live) {
        float h[8], a[8], g[8];
        unpack8(*reinterpret_cast<const uint4*>(dH + off), h);
        unpack8(*reinterpret_cast<const uint4*>(A + off), a);
        unpack8(*reinterpret_cast<const uint4*>(B + off), g);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float sg = sigmoid_(a[j]);
            const float silu = a[j] * sg;
            const float dsilu = sg * (1.0f + a[j] * (1.0f - sg));
            da[j] = h[j] * g[j] * dsilu;
            db[j] = h[j] * silu;
        }
        *reinterpret_cast<uint4*>(dA + off) = pack8(da);
        *reinterpret_cast<uint4*>(dB + off) = pack8(db);
    } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) da[j] = db[j] = 0.f;
    }
    const int ea = e8m0_exp_4lanes(da);
    const int eb = e8m0_exp_4lanes(db);
    if (!live) return;
    const int64_t qrow = r * 2 * F;
    *reinterpret_cast<uint2*>(q + qrow + 8 * c8) = encode8(da, ea);
    *reinterpret_cast<uint2*>(q + qrow + F + 8 * c8) = encode8(db, eb);
    if ((c8 & 3) == 0) {
        const int64_t srow = r * 2 * nb;
        s[srow + (c8 >> 2)] = (uint8_t)(ea + 127);
        s[srow + nb + (c8 >> 2)] = (uint8_t)(eb + 127);
    }
}

inline size_t a256(size_t n) { return (n + 255) & ~size_t(255); }

struct Carve {
    void* dYe;        // [R,d] bf16
    uint8_t* dYeq;    // [R,d]
    uint8_t* dYes;    // [R,d/32]
    uint8_t* dYesp;   // tile-packed (K = d)
    void* dH;         // [R,F] bf16; later deq(Hq)
    void* dA;         // [R,F] bf16
    void* dB;         // [R,F] bf16
    uint8_t* dABq;    // [R,2F]
    uint8_t* dABs;    // [R,2F/32]
    uint8_t* dABsp;   // tile-packed (K = 2F)
    void* dXe;        // [R,d] bf16; later deq(Xq)
    uint8_t* Hs;      // [R,F/32] row-layout H scales
    size_t total;
};

inline Carve carve(void* base, int64_t T, int64_t d, int64_t E, int64_t F, int k) {
    const size_t R = (size_t)T * (size_t)k;
    char* p = static_cast<char*>(base);
    size_t off = 0;
    auto take = [&](size_t n) {
        char* q = p + off;
        off += a256(n);
        return q;
    };
    Carve c;
    c.dYe = take(R * d * 2);
    c.dYeq = reinterpret_cast<uint8_t*>(take(R * d));
    c.dYes = reinterpret_cast<uint8_t*>(take(R * d / 32));
    c.dYesp = reinterpret_cast<uint8_t*>(take(mxfp8_act_scales_packed_size(E, (int64_t)R, d)));
    c.dH = take(R * F * 2);
    c.dA = take(R * F * 2);
    c.dB = take(R * F * 2);
    c.dABq = reinterpret_cast<uint8_t*>(take(R * 2 * F));
    c.dABs = reinterpret_cast<uint8_t*>(take(R * 2 * F / 32));
    c.dABsp = reinterpret_cast<uint8_t*>(take(mxfp8_act_scales_packed_size(E, (int64_t)R, 2 * F)));
    c.dXe = take(R * d * 2);
    c.Hs = reinterpret_cast<uint8_t*>(take(R * F / 32));
    c.total = off;
    return c;
}

}  // namespace mxb
}  // namespace moe

using namespace moe;

extern "C" int mxfp8_quantize_weights_bwd(const void* W1, const void* W3, const void* W2,
                                          int64_t w13_expert_stride, int64_t w2_expert_stride,
                                          int64_t E, int64_t d, int64_t F, uint8_t* W13tq,
                                          uint8_t* W13ts, uint8_t* W2tq, uint8_t* W2ts,
                                          void* stream) {
    if (E < 1 || E > MOE_MAX_EXPERTS || d <= 0 || F <= 0) return MOE_ERR_INVALID;
    if (d % 128 != 0 || F % 128 != 0 || d > (1 << 20) || F > (1 << 20)) return MOE_ERR_UNSUPPORTED;
    const void* ptrs[] = {W1, W3, W2, W13tq, W13ts, W2tq, W2ts};
    for (const void* p : ptrs)
        if (!p || !aligned16(p)) return MOE_ERR_INVALID;
    if ((w13_expert_stride < F * d || w2_expert_stride < F * d) && E > 1) return MOE_ERR_INVALID;
    if (w13_expert_stride < 0 || w2_expert_stride < 0) return MOE_ERR_INVALID;
    if (check_only()) return MOE_OK;
    cudaStream_t st = as_stream(stream);
    // W1_e, W3_e [F, d] -> rows i of [E, d, 2F]: (W1_e[:, i] | W3_e[:, i]) along F
    int rc = mxb::transpose_quant(W1, w13_expert_stride, E, F, d, W13tq, W13ts, 2 * F, 0, st);
    if (rc != MOE_OK) return rc;
    rc = mxb::transpose_quant(W3, w13_expert_stride, E, F, d, W13tq, W13ts, 2 * F, F, st);
    if (rc != MOE_OK) return rc;
    // W2_e [d, F] -> rows f of [E, F, d]: W2_e[:, f] along d
    return mxb::transpose_quant(W2, w2_expert_stride, E, d, F, W2tq, W2ts, d, 0, st);
}

extern "C" int moe_swiglu_bwd_mxfp8(const void* dH, const void* A, const void* B, int64_t R,
                                    int64_t F, void* dA, void* dB, uint8_t* dABq, uint8_t* dABs,
                                    void* stream) {
    if (R < 0 || F <= 0 || F % 32 != 0 || F > (1 << 24)) return MOE_ERR_INVALID;
    if (R == 0) return MOE_OK;
    const void* ptrs[] = {dH, A, B, dA, dB, dABq};
    for (const void* p : ptrs)
        if (!p || !aligned16(p)) return MOE_ERR_INVALID;
    if (!dABs) return MOE_ERR_INVALID;
    const int64_t n = R * (F / 8);  // one thread per 8 columns
    const int64_t blocks = (n + 255) / 256;
    if (blocks > INT32_MAX) return MOE_ERR_UNSUPPORTED;
    if (check_only()) return MOE_OK;
    mxb::swiglu_bwd_quant_kernel<<<(unsigned)blocks, 256, 0, as_stream(stream)>>>(
        static_cast<const __nv_bfloat16*>(dH), static_cast<const __nv_bfloat16*>(A),
        static_cast<const __nv_bfloat16*>(B), R, (int)F, static_cast<__nv_bfloat16*>(dA),
        static_cast<__nv_bfloat16*>(dB), dABq, dABs);
    return launch_status();
}

extern "C" size_t moe_layer_bwd_mxfp8_workspace_size(int64_t T, int64_t d, int64_t E, int64_t F,
                                                     int k) {
    if (T < 0 || d <= 0 || E <= 0 || F <= 0 || k <= 0) return 0;
    return mxb::carve(nullptr, T, d, E, F, k).total;
}

namespace moe {
namespace mxb {
static int bwd_steps(const moe_layer_bwd_mxfp8_args* a, const Carve& c, void* stream);
}  // namespace mxb
}  // namespace moe

extern "C" int moe_layer_bwd_mxfp8(const moe_layer_bwd_mxfp8_args* a, void* stream) {
    if (!a) return MOE_ERR_INVALID;
    if (a->T < 0 || a->d <= 0 || a->E < 1 || a->E > MOE_MAX_EXPERTS || a->F <= 0 || a->k < 1 ||
        a->k > a->E)
        return MOE_ERR_INVALID;
    if (a->d % 256 != 0 || a->F % 256 != 0) return MOE_ERR_UNSUPPORTED;
    if (!a->workspace || (reinterpret_cast<uintptr_t>(a->workspace) & 255u) != 0)
        return MOE_ERR_INVALID;
    const mxb::Carve c = mxb::carve(a->workspace, a->T, a->d, a->E, a->F, a->k);
    if (a->workspace_bytes < c.total) return MOE_ERR_INVALID;
    const void* need[] = {a->slot, a->gate, a->offsets, a->Xq, a->Xs, a->Hq, a->Hsp, a->A, a->B,
                          a->W13tq, a->Ps13t, a->W2tq, a->Ps2t, a->dOut, a->dx, a->dW1, a->dW3,
                          a->dW2};
    for (const void* p : need)
        if (!p) return MOE_ERR_INVALID;
    // what the steps below check, checked before the first launch
    const void* rows[] = {a->Xq, a->Hq, a->Hsp, a->A, a->B, a->W13tq, a->Ps13t, a->W2tq, a->Ps2t,
                          a->dOut, a->dx, a->dW1, a->dW3, a->dW2};
    for (const void* p : rows)
        if (!aligned16(p)) return MOE_ERR_INVALID;
    if (a->T * a->k > INT32_MAX - 256 || a->d > (1 << 24) || 2 * a->F > (1 << 24))
        return MOE_ERR_UNSUPPORTED;
    return checked([&] { return mxb::bwd_steps(a, c, stream); });
}

namespace moe {
namespace mxb {

// The steps of moe_layer_bwd_mxfp8 after its own checks.
static int bwd_steps(const moe_layer_bwd_mxfp8_args* a, const Carve& c, void* stream) {
    const int64_t T = a->T, d = a->d, E = a->E, F = a->F, R = a->T * a->k;
    int rc;
    if (R > 0) {
        // dYe = bf16(gate * dOut[t]) at each slot, then its MXFP8 codes along d
        rc = moe_dispatch(a->dOut, a->slot, a->gate, T, d, a->k, MOE_BF16, c.dYe, stream);
        if (rc != MOE_OK) return rc;
        rc = mxfp8_quantize(c.dYe, MOE_BF16, R, d, MOE_SCALE_E8M0, c.dYeq, c.dYes, stream);
        if (rc != MOE_OK) return rc;
        rc = mxfp8_pack_act_scales(c.dYes, a->offsets, E, R, d, c.dYesp, stream);
        if (rc != MOE_OK) return rc;
        // dH [R, F] = Q(dYe) Q(W2_e along d)ᵀ: the down GEMM with K = d, N = F
        rc = moe_grouped_down_mxfp8(c.dYeq, c.dYesp, a->W2tq, a->Ps2t, F * d, a->offsets, E, R,
                                    F, d, c.dH, stream);
        if (rc != MOE_OK) return rc;
        rc = moe_swiglu_bwd_mxfp8(c.dH, a->A, a->B, R, F, c.dA, c.dB, c.dABq, c.dABs, stream);
        if (rc != MOE_OK) return rc;
        rc = mxfp8_pack_act_scales(c.dABs, a->offsets, E, R, 2 * F, c.dABsp, stream);
        if (rc != MOE_OK) return rc;
        // dXe [R, d] = Q([dA | dB]) Q([W1_e; W3_e] along F): K = 2F, N = d
        rc = moe_grouped_down_mxfp8(c.dABq, c.dABsp, a->W13tq, a->Ps13t, d * 2 * F, a->offsets, E,
                                    R, d, 2 * F, c.dXe, stream);
        if (rc != MOE_OK) return rc;
        rc = moe_combine(c.dXe, a->slot, nullptr, T, d, a->k, MOE_BF16, a->dx, stream);
        if (rc != MOE_OK) return rc;
        // the forward's operands, dequantised (exact in bf16), for the weight gradients
        rc = mxfp8_dequantize(a->Xq, a->Xs, MOE_SCALE_E8M0, R, d, c.dXe, stream);
        if (rc != MOE_OK) return rc;
        rc = mxfp8_unpack_act_scales(a->Hsp, a->offsets, E, R, F, c.Hs, stream);
        if (rc != MOE_OK) return rc;
        rc = mxfp8_dequantize(a->Hq, c.Hs, MOE_SCALE_E8M0, R, F, c.dH, stream);
        if (rc != MOE_OK) return rc;
    }
    return swiglu_wgrad(c.dXe, c.dA, c.dB, c.dYe, c.dH, a->offsets, E, R, d, F, a->dW1, a->dW3,
                        a->dW2, as_stream(stream));
}

}  // namespace mxb
}  // namespace moe
