// Router backward and the load-balancing auxiliary loss of the dropless
// top-k MoE layer (sm_100a).
//
// "Transformers 中的 OLMoE" (blog.gitcode.com) §2: gates are the fp32 softmax
// probabilities of the top-k experts (optionally renormalised over the k);
// §4 "负载均衡辅助损失": a Switch-Transformer-style loss from the per-expert
// assignment frequency and the mean routing probability, multiplied and
// summed, scaled into the total loss by router_aux_loss_coef.
//
//   aux        = E * sum_e (counts[e]/T) * (1/T) sum_t p[t,e]
//   dgate[t,j] = <dOut[t], Ye[slot[t,j]]>           (out = sum_j gate * Ye)
//   dp[t,e]    = sum_j [idx[t,j]==e] dsel[t,j] + aux_coef * E * counts[e]/T^2
//                dsel = dgate, or with renormalised gates g = p_sel/S:
//                dsel = (dgate - sum_i g_i dgate_i) / S
//   dlogits    = p * (dp - sum_e p dp)              (softmax Jacobian)
//   logits = x Wr^T:  dx += dlogits Wr,  dWr = dlogits^T x
// The top-k choice and the counts are piecewise constant and get no
// gradient.
//
// gate_grad_kernel: one CTA per token (grid stride). The k dot products
// stream dOut[t] and the k rows Ye[slot[t,j]] in 16-byte vectors (HBM-bound,
// like the combine) and reduce over the block in a fixed order.
// softmax_bwd_kernel: one warp per token recomputes the token's fp32 softmax
// and applies the renorm backward, the aux term and the softmax Jacobian.
// aux: per-block column sums of p over token ranges, then one block sums
// them in a fixed order; no atomics, so every result is deterministic.
// Router GEMM backward: fp32 CUDA-core tiles (E is small, K = E for dx);
// dWr reduces over T in fixed token chunks into a workspace, then sums the
// chunks in order.
#include "common.cuh"

namespace moe {
namespace rb {

constexpr int THREADS = 256;
constexpr int WARPS = THREADS / 32;
constexpr int JB = 8;           // expert rows in flight per thread
constexpr int EPL_MAX = MOE_MAX_EXPERTS / 32;  // logits per lane, aux kernel
constexpr int AUX_MAX_BLOCKS = 128;
constexpr int AUX_TOKENS_MIN = 64;

template <int DT>
struct Vec;
template <>
struct Vec<MOE_BF16> {
    static constexpr int N = 8;
    __device__ static void load(const uint4& u, float* f) { unpack8(u, f); }
};
template <>
struct Vec<MOE_F32> {
    static constexpr int N = 4;
    __device__ static void load(const uint4& u, float* f) {
        f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y);
        f[2] = __uint_as_float(u.z); f[3] = __uint_as_float(u.w);
    }
};

// dg[t * dg_stride + j] = <dOut[t], Ye[slot[t,j]]>. One CTA per token (grid
// stride); each thread keeps JB expert rows in flight and the block reduces
// the k sums in a fixed order (lanes, then warps).
template <int DT>
__global__ void __launch_bounds__(THREADS)
    gate_grad_kernel(const uint4* __restrict__ dOut, const uint4* __restrict__ Ye,
                     const int32_t* __restrict__ slot, int T, int vpr, int k, int64_t R,
                     float* __restrict__ dg, int dg_stride, int* status) {
    constexpr int N = Vec<DT>::N;
    __shared__ int s_slot[MOE_MAX_TOPK];
    __shared__ float s_part[WARPS][MOE_MAX_TOPK];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    for (int t = blockIdx.x; t < T; t += gridDim.x) {
        __syncthreads();
        if (tid < k) {
            int s = slot[(size_t)t * k + tid];
            if (s < 0 || s >= R) {
                set_status(status, MOE_DEVERR_BAD_INDEX);
                s = -1;
            }
            s_slot[tid] = s;
        }
        __syncthreads();
        for (int j0 = 0; j0 < k; j0 += JB) {
            float acc[JB];
#pragma unroll
            for (int jj = 0; jj < JB; ++jj) acc[jj] = 0.f;
            for (int v = tid; v < vpr; v += THREADS) {
                float g[N];
                Vec<DT>::load(__ldcs(dOut + (size_t)t * vpr + v), g);
                uint4 val[JB];
#pragma unroll
                for (int jj = 0; jj < JB; ++jj) {
                    const int j = j0 + jj;
                    const int s = j < k ? s_slot[j] : -1;
                    if (s >= 0) val[jj] = __ldcs(Ye + (size_t)s * vpr + v);
                }
#pragma unroll
                for (int jj = 0; jj < JB; ++jj) {
                    const int j = j0 + jj;
                    if (j >= k || s_slot[j] < 0) continue;
                    float y[N];
                    Vec<DT>::load(val[jj], y);
#pragma unroll
                    for (int q = 0; q < N; ++q) acc[jj] = fmaf(g[q], y[q], acc[jj]);
                }
            }
#pragma unroll
            for (int jj = 0; jj < JB; ++jj) {
                const float w = warp_sum(acc[jj]);
                if (lane == 0 && j0 + jj < k) s_part[warp][j0 + jj] = w;
            }
        }
        __syncthreads();
        if (tid < k) {
            float v = 0.f;
#pragma unroll
            for (int w = 0; w < WARPS; ++w) v += s_part[w][tid];
            dg[(size_t)t * dg_stride + tid] = v;
        }
    }
}

// One warp per token: the token's fp32 softmax, the gradient reaching the
// chosen probabilities (renorm backward if asked), the aux-loss term, and
// the softmax Jacobian. Lane l holds experts l, l + 32, ... (EPL of them).
// dg may alias dlogits (row t, stride E): a warp reads its token's k values
// before it writes that row, and touches no other row.
template <int EPL>
__global__ void __launch_bounds__(THREADS)
    softmax_bwd_kernel(const float* __restrict__ logits, const int32_t* __restrict__ idx,
                       const int32_t* __restrict__ counts, const float* dg, int dg_stride,
                       int T, int E, int k, int renorm, float aux_scale, float* dlogits,
                       int* status) {
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * WARPS + (threadIdx.x >> 5);
    if (t >= T) return;
    int e_j = -1;
    float dg_j = 0.f;
    if (lane < k) {
        e_j = idx[(size_t)t * k + lane];
        if (e_j < 0 || e_j >= E) {
            set_status(status, MOE_DEVERR_BAD_INDEX);
            e_j = -1;
        }
        dg_j = dg[(size_t)t * dg_stride + lane];
    }
    __syncwarp();
    const float* lrow = logits + (size_t)t * E;
    float p[EPL];
    float mx = -INFINITY;
#pragma unroll
    for (int q = 0; q < EPL; ++q) {
        const int e = lane + 32 * q;
        p[q] = e < E ? lrow[e] : -INFINITY;
        mx = fmaxf(mx, p[q]);
    }
    mx = warp_max(mx);
    float sum = 0.f;
#pragma unroll
    for (int q = 0; q < EPL; ++q) {
        const int e = lane + 32 * q;
        p[q] = e < E ? expf(p[q] - mx) : 0.f;
        sum += p[q];
    }
    const float inv = 1.0f / warp_sum(sum);
#pragma unroll
    for (int q = 0; q < EPL; ++q) p[q] *= inv;
    float dsel = dg_j;
    if (renorm) {
        const float psel = e_j >= 0 ? expf(lrow[e_j] - mx) * inv : 0.f;
        const float S = warp_sum(psel);
        const float gdot = warp_sum(lane < k ? (psel / S) * dg_j : 0.f);
        dsel = (dg_j - gdot) / S;
    }
    float dp[EPL];
    float pdp = 0.f;
#pragma unroll
    for (int q = 0; q < EPL; ++q) {
        const int e = lane + 32 * q;
        float v = (aux_scale != 0.f && e < E) ? aux_scale * (float)counts[e] : 0.f;
        for (int j = 0; j < k; ++j) {
            const int ej = __shfl_sync(0xffffffffu, e_j, j);
            const float dj = __shfl_sync(0xffffffffu, dsel, j);
            if (ej == e) v += dj;
        }
        dp[q] = e < E ? v : 0.f;
        pdp = fmaf(p[q], dp[q], pdp);
    }
    pdp = warp_sum(pdp);
#pragma unroll
    for (int q = 0; q < EPL; ++q) {
        const int e = lane + 32 * q;
        if (e < E) dlogits[(size_t)t * E + e] = p[q] * (dp[q] - pdp);
    }
}

// Column sums of softmax(logits) over a token range, one block per range:
// warp w takes tokens w, w + WARPS, ...; the warps' sums are added in warp
// order into partial[block][e].
__global__ void __launch_bounds__(THREADS)
    aux_partial_kernel(const float* __restrict__ logits, int T, int E, int tokens_per_block,
                       float* __restrict__ partial) {
    __shared__ float s_col[WARPS][MOE_MAX_EXPERTS];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int t0 = blockIdx.x * tokens_per_block;
    const int t1 = min(T, t0 + tokens_per_block);
    float colsum[EPL_MAX];
#pragma unroll
    for (int q = 0; q < EPL_MAX; ++q) colsum[q] = 0.f;
    for (int t = t0 + warp; t < t1; t += WARPS) {
        const float* lrow = logits + (size_t)t * E;
        float p[EPL_MAX];
        float mx = -INFINITY;
#pragma unroll
        for (int q = 0; q < EPL_MAX; ++q) {
            const int e = lane + 32 * q;
            p[q] = e < E ? lrow[e] : -INFINITY;
            mx = fmaxf(mx, p[q]);
        }
        mx = warp_max(mx);
        float sum = 0.f;
#pragma unroll
        for (int q = 0; q < EPL_MAX; ++q) {
            const int e = lane + 32 * q;
            p[q] = e < E ? expf(p[q] - mx) : 0.f;
            sum += p[q];
        }
        const float inv = 1.0f / warp_sum(sum);
#pragma unroll
        for (int q = 0; q < EPL_MAX; ++q) colsum[q] += p[q] * inv;
    }
#pragma unroll
    for (int q = 0; q < EPL_MAX; ++q) {
        const int e = lane + 32 * q;
        if (e < E) s_col[warp][e] = colsum[q];
    }
    __syncthreads();
    for (int e = tid; e < E; e += THREADS) {
        float v = 0.f;
#pragma unroll
        for (int w = 0; w < WARPS; ++w) v += s_col[w][e];
        partial[(size_t)blockIdx.x * E + e] = v;
    }
}

// aux = E * sum_e (counts[e]/T) * (P_sum[e]/T). Thread e adds the partials
// of expert e over the blocks in block order (loads issued 16 at a time,
// coalesced across experts), then the expert terms are added in a fixed
// shared-memory tree, so the result is deterministic.
constexpr int AUX_FINAL_THREADS = MOE_MAX_EXPERTS;

__global__ void __launch_bounds__(AUX_FINAL_THREADS)
    aux_final_kernel(const float* __restrict__ partial, int nblocks,
                     const int32_t* __restrict__ counts, int T, int E, float* __restrict__ aux) {
    __shared__ float s_red[AUX_FINAL_THREADS];
    const int e = threadIdx.x;
    float term = 0.f;
    if (e < E) {
        float P = 0.f;
        int b = 0;
        for (; b + 16 <= nblocks; b += 16) {
            float v[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] = partial[(size_t)(b + i) * E + e];
#pragma unroll
            for (int i = 0; i < 16; ++i) P += v[i];
        }
        for (; b < nblocks; ++b) P += partial[(size_t)b * E + e];
        term = (float)counts[e] * P;
    }
    s_red[e] = term;
    __syncthreads();
    for (int w = AUX_FINAL_THREADS / 2; w > 0; w >>= 1) {
        if (e < w) s_red[e] += s_red[e + w];
        __syncthreads();
    }
    if (e == 0) {
        const float invT = 1.0f / (float)T;
        aux[0] = (float)E * s_red[0] * invT * invT;
    }
}

inline int aux_blocks(int64_t T) {
    int64_t b = (T + AUX_TOKENS_MIN - 1) / AUX_TOKENS_MIN;
    return (int)(b < AUX_MAX_BLOCKS ? (b < 1 ? 1 : b) : AUX_MAX_BLOCKS);
}

// ---------------------------------------------------------------- router GEMMs

constexpr int LT = 64;   // tokens (dx) or experts (dWr) per tile
constexpr int LC = 128;  // columns of d per tile
constexpr int LK = 32;   // contraction chunk staged in shared memory

template <typename TX>
__device__ __forceinline__ float to_f(TX v);
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }
template <>
__device__ __forceinline__ float to_f<float>(float v) { return v; }

template <typename TX>
__device__ __forceinline__ TX from_f(float v);
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }
template <>
__device__ __forceinline__ float from_f<float>(float v) { return v; }

// dx[t, c] = round(dx[t, c] + sum_e dlogits[t, e] * Wr[e, c]), fp32 sum over
// e in ascending order. Thread (g = tid/32, l = tid%32) owns tokens 8g..8g+7
// and columns 4l..4l+3 of a 64 x 128 tile; a warp shares its tokens, so
// the dlogits reads are broadcasts and the Wr reads are 16-byte vectors.
template <typename TX>
__global__ void __launch_bounds__(THREADS)
    router_dx_kernel(const float* __restrict__ dlogits, const TX* __restrict__ Wr, int T, int d,
                     int E, TX* __restrict__ dx) {
    __shared__ float s_dl[LT][LK + 1];
    __shared__ __align__(16) float s_w[LK][LC];
    const int tid = threadIdx.x, g = tid >> 5, l = tid & 31;
    const int t0 = blockIdx.x * LT, c0 = blockIdx.y * LC;
    float acc[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
    for (int e0 = 0; e0 < E; e0 += LK) {
        __syncthreads();
        for (int i = tid; i < LT * LK; i += THREADS) {
            const int r = i / LK, e = i % LK;
            const int t = t0 + r;
            s_dl[r][e] = (t < T && e0 + e < E) ? dlogits[(size_t)t * E + e0 + e] : 0.f;
        }
        for (int i = tid; i < LK * LC; i += THREADS) {
            const int e = i / LC, c = i % LC;
            s_w[e][c] = (e0 + e < E && c0 + c < d) ? to_f(Wr[(size_t)(e0 + e) * d + c0 + c]) : 0.f;
        }
        __syncthreads();
#pragma unroll 4
        for (int e = 0; e < LK; ++e) {
            const float4 b = *reinterpret_cast<const float4*>(&s_w[e][4 * l]);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float a = s_dl[8 * g + i][e];
                acc[i][0] = fmaf(a, b.x, acc[i][0]);
                acc[i][1] = fmaf(a, b.y, acc[i][1]);
                acc[i][2] = fmaf(a, b.z, acc[i][2]);
                acc[i][3] = fmaf(a, b.w, acc[i][3]);
            }
        }
    }
    const int c = c0 + 4 * l;
    if (c >= d) return;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int t = t0 + 8 * g + i;
        if (t >= T) continue;
        TX* row = dx + (size_t)t * d + c;
#pragma unroll
        for (int j = 0; j < 4; ++j) row[j] = from_f<TX>(to_f(row[j]) + acc[i][j]);
    }
}

// partial[ch][e][c] = sum over the chunk's tokens (ascending) of
// dlogits[t, e] * x[t, c]. Thread (g, l) owns experts 8g..8g+7 and columns
// 4l..4l+3 of a 64 x 128 tile.
template <typename TX>
__global__ void __launch_bounds__(THREADS)
    router_dwr_partial_kernel(const float* __restrict__ dlogits, const TX* __restrict__ x, int T,
                              int d, int E, int tokens_per_chunk, float* __restrict__ partial) {
    __shared__ float s_dl[LK][LT + 1];
    __shared__ __align__(16) float s_x[LK][LC];
    const int tid = threadIdx.x, g = tid >> 5, l = tid & 31;
    const int ch = blockIdx.x, e0 = blockIdx.y * LT, c0 = blockIdx.z * LC;
    const int tb = ch * tokens_per_chunk, te = min(T, tb + tokens_per_chunk);
    float acc[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
    for (int s0 = tb; s0 < te; s0 += LK) {
        __syncthreads();
        for (int i = tid; i < LK * LT; i += THREADS) {
            const int r = i / LT, e = i % LT;
            const int t = s0 + r;
            s_dl[r][e] = (t < te && e0 + e < E) ? dlogits[(size_t)t * E + e0 + e] : 0.f;
        }
        for (int i = tid; i < LK * LC; i += THREADS) {
            const int r = i / LC, c = i % LC;
            const int t = s0 + r;
            s_x[r][c] = (t < te && c0 + c < d) ? to_f(x[(size_t)t * d + c0 + c]) : 0.f;
        }
        __syncthreads();
#pragma unroll 4
        for (int r = 0; r < LK; ++r) {
            const float4 b = *reinterpret_cast<const float4*>(&s_x[r][4 * l]);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float a = s_dl[r][8 * g + i];
                acc[i][0] = fmaf(a, b.x, acc[i][0]);
                acc[i][1] = fmaf(a, b.y, acc[i][1]);
                acc[i][2] = fmaf(a, b.z, acc[i][2]);
                acc[i][3] = fmaf(a, b.w, acc[i][3]);
            }
        }
    }
    const int c = c0 + 4 * l;
    if (c >= d) return;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int e = e0 + 8 * g + i;
        if (e >= E) continue;
        float4* dst = reinterpret_cast<float4*>(partial + ((size_t)ch * E + e) * d + c);
        *dst = make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
    }
}

// dWr[e, c] = round(sum over chunks, in order, of partial[ch][e][c])
template <typename TX>
__global__ void __launch_bounds__(THREADS)
    router_dwr_reduce_kernel(const float* __restrict__ partial, int nchunks, int64_t n,
                             TX* __restrict__ dWr) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        float v = 0.f;
        for (int ch = 0; ch < nchunks; ++ch) v += partial[(size_t)ch * n + i];
        dWr[i] = from_f<TX>(v);
    }
}

// Token chunks of the dWr reduction: enough (expert tile, column tile,
// chunk) blocks for about 4 x 148 CTAs, each chunk a multiple of LK tokens,
// at most 64 chunks. A function of the sizes only, so the workspace size is
// known on the host.
struct DwrSplit {
    int chunks, tokens;
};
inline DwrSplit dwr_split(int64_t T, int64_t d, int64_t E) {
    const int64_t tiles = ((E + LT - 1) / LT) * ((d + LC - 1) / LC);
    int64_t want = (592 + tiles - 1) / tiles;
    if (want > 64) want = 64;
    if (want < 1) want = 1;
    int64_t tok = (T + want - 1) / want;
    tok = (tok + LK - 1) / LK * LK;
    if (tok < LK) tok = LK;
    DwrSplit s;
    s.tokens = (int)tok;
    s.chunks = (int)((T + tok - 1) / tok);
    if (s.chunks < 1) s.chunks = 1;
    return s;
}

// ---------------------------------------------------------------- tensor-core path
//
// bf16 router GEMM backward on the tensor cores (the router is a linear
// layer in the model's dtype, "Transformers 中的 OLMoE" §2, and its backward
// runs in that dtype too): dlogits is rounded to bf16 once, then dx += dl Wr
// and the partials of dWr = dlᵀ x over token chunks are tcgen05 GEMMs with
// fp32 accumulation (backward.cu), and the chunks are summed in order as on
// the CUDA-core path. Used when d % 256 == 0.
constexpr int TC_CHUNK_MIN = 512;  // tokens per dWr chunk (at most MOE_MAX_EXPERTS chunks)

struct TcLayout {
    int64_t Ep, Mp, chunk, G;
    size_t off_one, off_chunks, dl, partial, total;
};

inline size_t align256(size_t b) { return (b + 255) & ~size_t(255); }

inline TcLayout tc_layout(int64_t T, int64_t d, int64_t E) {
    TcLayout L;
    L.Ep = (E + 63) / 64 * 64;
    L.Mp = (E + 127) / 128 * 128;
    int64_t chunk = (T + MOE_MAX_EXPERTS - 1) / MOE_MAX_EXPERTS;
    chunk = (chunk + 63) / 64 * 64;
    L.chunk = chunk < TC_CHUNK_MIN ? TC_CHUNK_MIN : chunk;
    L.G = T > 0 ? (T + L.chunk - 1) / L.chunk : 1;
    L.off_one = 0;
    L.off_chunks = 256;
    L.dl = L.off_chunks + align256(sizeof(int32_t) * (size_t)(MOE_MAX_EXPERTS + 1));
    L.partial = L.dl + align256(sizeof(uint16_t) * (size_t)T * (size_t)L.Ep);
    L.total = L.partial + sizeof(float) * (size_t)L.G * (size_t)L.Mp * (size_t)d;
    return L;
}

// dl[t, e] = bf16(dlogits[t, e]) for e < E, 0 for E <= e < Ep; the row-group
// offsets {0, T} and the chunk offsets {0, chunk, 2 chunk, ..., T}.
__global__ void __launch_bounds__(THREADS)
    dl_to_bf16_kernel(const float* __restrict__ dlogits, int64_t T, int E, int Ep, int G,
                      int chunk, __nv_bfloat16* __restrict__ dl, int32_t* __restrict__ off_one,
                      int32_t* __restrict__ off_chunks) {
    const int64_t n = T * Ep;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = i / Ep;
        const int e = (int)(i - t * Ep);
        dl[i] = __float2bfloat16_rn(e < E ? dlogits[t * E + e] : 0.f);
    }
    if (blockIdx.x == 0) {
        if (threadIdx.x == 0) {
            off_one[0] = 0;
            off_one[1] = (int32_t)T;
        }
        for (int g = threadIdx.x; g <= G; g += blockDim.x)
            off_chunks[g] = (int32_t)((int64_t)g * chunk < T ? (int64_t)g * chunk : T);
    }
}

// dWr[e, c] = round(sum over chunks, in order, of partial[g][e][c]), partial
// rows Mp apart per chunk.
__global__ void __launch_bounds__(THREADS)
    dwr_reduce_pitched_kernel(const float* __restrict__ partial, int G, int64_t Mp, int E,
                              int64_t d, __nv_bfloat16* __restrict__ dWr) {
    const int64_t n = (int64_t)E * d;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t e = i / d, c = i - e * d;
        float v = 0.f;
        for (int g = 0; g < G; ++g) v += partial[((int64_t)g * Mp + e) * d + c];
        dWr[i] = __float2bfloat16_rn(v);
    }
}

}  // namespace rb

int router_linear_bwd_tc(const void* dl, int64_t Ep, const void* x, const void* Wr, int64_t T,
                         int64_t d, int64_t E, const int32_t* off_one, const int32_t* off_chunks,
                         int64_t G, int64_t Mp, void* dx, float* partial, cudaStream_t st);

}  // namespace moe

using namespace moe;

extern "C" size_t moe_aux_loss_workspace_size(int64_t T, int64_t E) {
    if (T < 0 || E < 1 || E > MOE_MAX_EXPERTS) return 0;
    return sizeof(float) * (size_t)rb::aux_blocks(T) * (size_t)E;
}

extern "C" int moe_aux_loss(const float* logits, const int32_t* counts, int64_t T, int64_t E,
                            float* aux_out, void* workspace, size_t workspace_bytes, void* stream) {
    if (T < 1 || E < 1 || E > MOE_MAX_EXPERTS || T > INT32_MAX) return MOE_ERR_INVALID;
    if (!logits || !counts || !aux_out || !workspace) return MOE_ERR_INVALID;
    if ((reinterpret_cast<uintptr_t>(workspace) & 15u) != 0) return MOE_ERR_INVALID;
    if (workspace_bytes < moe_aux_loss_workspace_size(T, E)) return MOE_ERR_INVALID;
    if (check_only()) return MOE_OK;
    const int nb = rb::aux_blocks(T);
    const int per = (int)((T + nb - 1) / nb);
    const int used = (int)((T + per - 1) / per);
    cudaStream_t st = as_stream(stream);
    float* part = static_cast<float*>(workspace);
    rb::aux_partial_kernel<<<used, rb::THREADS, 0, st>>>(logits, (int)T, (int)E, per, part);
    rb::aux_final_kernel<<<1, rb::AUX_FINAL_THREADS, 0, st>>>(part, used, counts, (int)T, (int)E,
                                                               aux_out);
    return launch_status();
}

extern "C" int moe_router_bwd(const void* dOut, const void* Ye, const int32_t* slot,
                              const int32_t* idx, const float* logits, const int32_t* counts,
                              int64_t T, int64_t d, int64_t E, int k, int dtype, int renorm,
                              float aux_coef, float* dgate, float* dlogits, void* stream) {
    if (T < 0 || d <= 0 || E < 1 || E > MOE_MAX_EXPERTS || k < 1 || k > E || k > MOE_MAX_TOPK)
        return MOE_ERR_INVALID;
    if (dtype != MOE_BF16 && dtype != MOE_F32) return MOE_ERR_UNSUPPORTED;
    const int es = dtype == MOE_F32 ? 4 : 2;
    if ((d * es) % 16 != 0) return MOE_ERR_UNSUPPORTED;
    if (T == 0) return MOE_OK;
    if (T * k > INT32_MAX || T * E > INT32_MAX) return MOE_ERR_UNSUPPORTED;
    if (!dOut || !Ye || !slot || !idx || !logits || !dlogits) return MOE_ERR_INVALID;
    if (!aligned16(dOut) || !aligned16(Ye)) return MOE_ERR_INVALID;
    if (aux_coef != 0.f && !counts) return MOE_ERR_INVALID;
    if (check_only()) return MOE_OK;
    const double aux_scale = (double)aux_coef * (double)E / ((double)T * (double)T);
    const int vpr = (int)(d * es / 16);
    int64_t g = T;
    const int64_t cap = (int64_t)num_sms() * 8;
    if (g > cap) g = cap;
    cudaStream_t st = as_stream(stream);
    // without a dgate output the gate gradients are parked in the first k
    // entries of each token's dlogits row
    float* dg = dgate ? dgate : dlogits;
    const int dg_stride = dgate ? k : (int)E;
    const uint4* o = static_cast<const uint4*>(dOut);
    const uint4* y = static_cast<const uint4*>(Ye);
    if (dtype == MOE_BF16)
        rb::gate_grad_kernel<MOE_BF16><<<(int)g, rb::THREADS, 0, st>>>(
            o, y, slot, (int)T, vpr, k, T * k, dg, dg_stride, status_ptr());
    else
        rb::gate_grad_kernel<MOE_F32><<<(int)g, rb::THREADS, 0, st>>>(
            o, y, slot, (int)T, vpr, k, T * k, dg, dg_stride, status_ptr());
    if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
    const int blocks = (int)((T + rb::WARPS - 1) / rb::WARPS);
    switch ((E + 31) / 32) {
#define MOE_SMBWD_CASE(n)                                                                      \
    case n:                                                                                    \
        rb::softmax_bwd_kernel<n><<<blocks, rb::THREADS, 0, st>>>(                             \
            logits, idx, counts, dg, dg_stride, (int)T, (int)E, k, renorm, (float)aux_scale,   \
            dlogits, status_ptr());                                                            \
        break;
        MOE_SMBWD_CASE(1) MOE_SMBWD_CASE(2) MOE_SMBWD_CASE(3) MOE_SMBWD_CASE(4)
        MOE_SMBWD_CASE(5) MOE_SMBWD_CASE(6) MOE_SMBWD_CASE(7) MOE_SMBWD_CASE(8)
        MOE_SMBWD_CASE(9) MOE_SMBWD_CASE(10) MOE_SMBWD_CASE(11) MOE_SMBWD_CASE(12)
        MOE_SMBWD_CASE(13) MOE_SMBWD_CASE(14) MOE_SMBWD_CASE(15) MOE_SMBWD_CASE(16)
#undef MOE_SMBWD_CASE
        default:
            return MOE_ERR_UNSUPPORTED;
    }
    return launch_status();
}

extern "C" size_t moe_router_linear_bwd_workspace_size(int64_t T, int64_t d, int64_t E) {
    if (T < 0 || d <= 0 || E < 1) return 0;
    const rb::DwrSplit s = rb::dwr_split(T, d, E);
    const size_t cuda_core = sizeof(float) * (size_t)s.chunks * (size_t)E * (size_t)d;
    const size_t tc = rb::tc_layout(T, d, E).total;
    return cuda_core > tc ? cuda_core : tc;
}

extern "C" int moe_router_linear_bwd(const float* dlogits, const void* x, const void* Wr,
                                     int64_t T, int64_t d, int64_t E, int dtype, void* dx,
                                     void* dWr, void* workspace, size_t workspace_bytes,
                                     void* stream) {
    if (T < 0 || d <= 0 || E < 1 || E > MOE_MAX_EXPERTS) return MOE_ERR_INVALID;
    if (dtype != MOE_BF16 && dtype != MOE_F32) return MOE_ERR_UNSUPPORTED;
    if (d % 4 != 0) return MOE_ERR_UNSUPPORTED;
    if (T > INT32_MAX / 2 || d > INT32_MAX / 2) return MOE_ERR_UNSUPPORTED;
    if (!dlogits) return MOE_ERR_INVALID;
    if (dx && !Wr) return MOE_ERR_INVALID;
    if (dWr && (!x || !workspace || (reinterpret_cast<uintptr_t>(workspace) & 15u) != 0 ||
                workspace_bytes < moe_router_linear_bwd_workspace_size(T, d, E)))
        return MOE_ERR_INVALID;
    if (check_only()) return MOE_OK;
    cudaStream_t st = as_stream(stream);
    const bool tc = dtype == MOE_BF16 && T > 0 && d % 256 == 0 && d <= (1 << 24) &&
                    T <= INT32_MAX - 2 * 128 && (!dx || (aligned16(dx) && aligned16(Wr))) &&
                    (!dWr || aligned16(x)) && workspace &&
                    (reinterpret_cast<uintptr_t>(workspace) & 255u) == 0 &&
                    workspace_bytes >= moe_router_linear_bwd_workspace_size(T, d, E);
    if (tc) {
        const rb::TcLayout L = rb::tc_layout(T, d, E);
        char* w = static_cast<char*>(workspace);
        int32_t* off_one = reinterpret_cast<int32_t*>(w + L.off_one);
        int32_t* off_chunks = reinterpret_cast<int32_t*>(w + L.off_chunks);
        __nv_bfloat16* dl = reinterpret_cast<__nv_bfloat16*>(w + L.dl);
        float* part = reinterpret_cast<float*>(w + L.partial);
        int64_t g = (T * L.Ep + rb::THREADS - 1) / rb::THREADS;
        const int64_t cap = (int64_t)num_sms() * 8;
        if (g > cap) g = cap;
        rb::dl_to_bf16_kernel<<<(int)g, rb::THREADS, 0, st>>>(dlogits, T, (int)E, (int)L.Ep,
                                                              (int)L.G, (int)L.chunk, dl,
                                                              off_one, off_chunks);
        int rc = router_linear_bwd_tc(dl, L.Ep, x, Wr, T, d, E, off_one, off_chunks, L.G, L.Mp,
                                      dx, dWr ? part : nullptr, st);
        if (rc != MOE_OK) return rc;
        if (dWr) {
            int64_t rg = (E * d + rb::THREADS - 1) / rb::THREADS;
            if (rg > cap) rg = cap;
            rb::dwr_reduce_pitched_kernel<<<(int)rg, rb::THREADS, 0, st>>>(
                part, (int)L.G, L.Mp, (int)E, d, static_cast<__nv_bfloat16*>(dWr));
        }
        return launch_status();
    }
    if (dx && T > 0) {
        const dim3 grid((unsigned)((T + rb::LT - 1) / rb::LT), (unsigned)((d + rb::LC - 1) / rb::LC));
        if (dtype == MOE_BF16)
            rb::router_dx_kernel<__nv_bfloat16><<<grid, rb::THREADS, 0, st>>>(
                dlogits, static_cast<const __nv_bfloat16*>(Wr), (int)T, (int)d, (int)E,
                static_cast<__nv_bfloat16*>(dx));
        else
            rb::router_dx_kernel<float><<<grid, rb::THREADS, 0, st>>>(
                dlogits, static_cast<const float*>(Wr), (int)T, (int)d, (int)E,
                static_cast<float*>(dx));
        if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
    }
    if (dWr) {
        const int64_t n = E * d;
        if (T == 0) {
            const size_t bytes = (size_t)n * (dtype == MOE_F32 ? 4 : 2);
            return cudaMemsetAsync(dWr, 0, bytes, st) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
        }
        const rb::DwrSplit s = rb::dwr_split(T, d, E);
        float* part = static_cast<float*>(workspace);
        const dim3 grid((unsigned)s.chunks, (unsigned)((E + rb::LT - 1) / rb::LT),
                        (unsigned)((d + rb::LC - 1) / rb::LC));
        int64_t rg = (n + rb::THREADS - 1) / rb::THREADS;
        const int64_t cap = (int64_t)num_sms() * 8;
        if (rg > cap) rg = cap;
        if (dtype == MOE_BF16) {
            rb::router_dwr_partial_kernel<__nv_bfloat16><<<grid, rb::THREADS, 0, st>>>(
                dlogits, static_cast<const __nv_bfloat16*>(x), (int)T, (int)d, (int)E, s.tokens,
                part);
            rb::router_dwr_reduce_kernel<__nv_bfloat16><<<(int)rg, rb::THREADS, 0, st>>>(
                part, s.chunks, n, static_cast<__nv_bfloat16*>(dWr));
        } else {
            rb::router_dwr_partial_kernel<float><<<grid, rb::THREADS, 0, st>>>(
                dlogits, static_cast<const float*>(x), (int)T, (int)d, (int)E, s.tokens, part);
            rb::router_dwr_reduce_kernel<float><<<(int)rg, rb::THREADS, 0, st>>>(
                part, s.chunks, n, static_cast<float*>(dWr));
        }
    }
    return launch_status();
}
