// Row-wise dispatch and gate-weighted combine of the dropless MoE layer.
//
// Dispatch ("olmoforge" README, capability table, row-wise expert
// parallelism): every (token, j) row goes straight to its slot of the
// expert-sorted buffer, Xe[slot[t,j]] = x[t]; one pass reads x[t] once and
// writes its k copies. Combine ("Transformers 中的 OLMoE" §3, multiply by the
// top-k weight and index_add_ back to the token): done as a gather per token,
// out[t] = sum_j gate[t,j] * Ye[slot[t,j]], fp32 fused multiply-add in
// ascending j, so no atomics and a deterministic result.
//
// Both kernels are HBM-bound streams of 16-byte vectors. A CTA walks tokens
// with a grid stride; each thread keeps UNROLL independent vectors in flight.
#include "common.cuh"

namespace moe {
namespace dc {

constexpr int THREADS = 256;
constexpr int UNROLL = 4;

// Elementwise helpers on 16-byte vectors for the scaled/accumulating paths.
template <int DT>
struct Vec;

template <>
struct Vec<MOE_BF16> {
    static constexpr int N = 8;
    __device__ static void load(const uint4& u, float* f) { unpack8(u, f); }
    __device__ static uint4 store(const float* f) { return pack8(f); }
};

template <>
struct Vec<MOE_F32> {
    static constexpr int N = 4;
    __device__ static void load(const uint4& u, float* f) {
        f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y);
        f[2] = __uint_as_float(u.z); f[3] = __uint_as_float(u.w);
    }
    __device__ static uint4 store(const float* f) {
        return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                          __float_as_uint(f[3]));
    }
};

// Xe[slot[t,j]] = x[t]   (SCALED: = round(gate[t,j] * x[t]));
// row_gate (if not null): row_gate[slot[t,j]] = gate[t,j], the gate of each
// expert row for the down GEMM's epilogue
template <int DT, bool SCALED>
__global__ void __launch_bounds__(THREADS) dispatch_kernel(const uint4* __restrict__ x,
                                                           const int32_t* __restrict__ slot,
                                                           const float* __restrict__ gate,
                                                           int T, int k, int vpr, int64_t R,
                                                           uint4* __restrict__ Xe, int* status,
                                                           float* __restrict__ row_gate) {
    __shared__ int s_slot[MOE_MAX_TOPK];
    __shared__ float s_gate[MOE_MAX_TOPK];
    for (int t = blockIdx.x; t < T; t += gridDim.x) {
        __syncthreads();
        if (threadIdx.x < k) {
            int s = slot[(size_t)t * k + threadIdx.x];
            if (s < 0 || s >= R) {
                set_status(status, MOE_DEVERR_BAD_INDEX);
                s = -1;
            }
            s_slot[threadIdx.x] = s;
            if (SCALED) s_gate[threadIdx.x] = gate[(size_t)t * k + threadIdx.x];
            if (row_gate != nullptr && s >= 0) row_gate[s] = gate[(size_t)t * k + threadIdx.x];
        }
        __syncthreads();
        const uint4* src = x + (size_t)t * vpr;
        for (int v0 = threadIdx.x; v0 < vpr; v0 += THREADS * UNROLL) {
            uint4 val[UNROLL];
#pragma unroll
            for (int u = 0; u < UNROLL; ++u) {
                const int v = v0 + u * THREADS;
                if (v < vpr) val[u] = __ldcs(src + v);
            }
            for (int j = 0; j < k; ++j) {
                const int s = s_slot[j];
                if (s < 0) continue;
                uint4* dst = Xe + (size_t)s * vpr;
#pragma unroll
                for (int u = 0; u < UNROLL; ++u) {
                    const int v = v0 + u * THREADS;
                    if (v >= vpr) continue;
                    if (SCALED) {
                        float f[Vec<DT>::N];
                        Vec<DT>::load(val[u], f);
                        const float g = s_gate[j];
#pragma unroll
                        for (int q = 0; q < Vec<DT>::N; ++q) f[q] = g * f[q];
                        dst[v] = Vec<DT>::store(f);
                    } else {
                        dst[v] = val[u];
                    }
                }
            }
        }
    }
}

// out[t] = sum_j gate[t,j] * Ye[slot[t,j]]  (UNIT: gate == 1)
// Each thread owns one 16-byte column vector of a token and issues the loads
// of up to JB rows before it accumulates them, so JB loads are in flight per
// thread; the accumulation itself stays in ascending j.
template <int DT, bool UNIT>
__global__ void __launch_bounds__(THREADS) combine_kernel(const uint4* __restrict__ Ye,
                                                          const int32_t* __restrict__ slot,
                                                          const float* __restrict__ gate, int T,
                                                          int k, int vpr, int64_t R,
                                                          uint4* __restrict__ out, int* status) {
    constexpr int JB = 8;
    __shared__ int s_slot[MOE_MAX_TOPK];
    __shared__ float s_gate[MOE_MAX_TOPK];
    constexpr int N = Vec<DT>::N;
    for (int t = blockIdx.x; t < T; t += gridDim.x) {
        __syncthreads();
        if (threadIdx.x < k) {
            int s = slot[(size_t)t * k + threadIdx.x];
            if (s < 0 || s >= R) {
                set_status(status, MOE_DEVERR_BAD_INDEX);
                s = -1;
            }
            s_slot[threadIdx.x] = s;
            s_gate[threadIdx.x] = UNIT ? 1.f : gate[(size_t)t * k + threadIdx.x];
        }
        __syncthreads();
        for (int v = threadIdx.x; v < vpr; v += THREADS) {
            float acc[N];
#pragma unroll
            for (int q = 0; q < N; ++q) acc[q] = 0.f;
            for (int j0 = 0; j0 < k; j0 += JB) {
                uint4 val[JB];
#pragma unroll
                for (int jj = 0; jj < JB; ++jj) {
                    const int j = j0 + jj;
                    const int s = (j < k) ? s_slot[j] : -1;
                    if (s >= 0) val[jj] = __ldcs(Ye + (size_t)s * vpr + v);
                }
#pragma unroll
                for (int jj = 0; jj < JB; ++jj) {
                    const int j = j0 + jj;
                    if (j >= k || s_slot[j] < 0) continue;
                    const float g = s_gate[j];
                    float f[N];
                    Vec<DT>::load(val[jj], f);
#pragma unroll
                    for (int q = 0; q < N; ++q) acc[q] = fmaf(g, f[q], acc[q]);
                }
            }
            out[(size_t)t * vpr + v] = Vec<DT>::store(acc);
        }
    }
}

// row_token[slot[t,j]] = t: the token whose copy each expert row holds (the
// inverse of the slot permutation), so a GEMM can fetch its A rows from x.
__global__ void __launch_bounds__(THREADS) row_token_kernel(const int32_t* __restrict__ slot,
                                                            int64_t n, int k, int64_t R,
                                                            int32_t* __restrict__ row_token,
                                                            int* status) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int s = slot[i];
        if (s < 0 || s >= R) {
            set_status(status, MOE_DEVERR_BAD_INDEX);
            continue;
        }
        row_token[s] = (int32_t)(i / k);
    }
}

inline int grid_for(int64_t T) {
    const int64_t cap = (int64_t)num_sms() * 8;
    return (int)(T < cap ? T : cap);
}

}  // namespace dc
}  // namespace moe

using namespace moe;

static int dispatch_impl(const void* x, const int32_t* slot, const float* gate, bool scaled,
                         int64_t T, int64_t d, int k, int dtype, void* Xe, float* row_gate,
                         void* stream) {
    if (T < 0 || d <= 0 || k < 1 || k > MOE_MAX_TOPK) return MOE_ERR_INVALID;
    if (dtype != MOE_F32 && dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
    const int es = dtype == MOE_F32 ? 4 : 2;
    if ((d * es) % 16 != 0) return MOE_ERR_UNSUPPORTED;
    if (T == 0) return MOE_OK;
    if (!x || !slot || !Xe || !aligned16(x) || !aligned16(Xe)) return MOE_ERR_INVALID;
    if (T * k > INT32_MAX) return MOE_ERR_UNSUPPORTED;
    if (check_only()) return MOE_OK;
    const int vpr = (int)(d * es / 16);
    const int64_t R = T * k;
    cudaStream_t st = as_stream(stream);
    const int grid = dc::grid_for(T);
    const uint4* xs = static_cast<const uint4*>(x);
    uint4* xe = static_cast<uint4*>(Xe);
    if (dtype == MOE_BF16) {
        if (scaled)
            dc::dispatch_kernel<MOE_BF16, true><<<grid, dc::THREADS, 0, st>>>(xs, slot, gate, (int)T, k, vpr, R, xe, status_ptr(), row_gate);
        else
            dc::dispatch_kernel<MOE_BF16, false><<<grid, dc::THREADS, 0, st>>>(xs, slot, gate, (int)T, k, vpr, R, xe, status_ptr(), row_gate);
    } else {
        if (scaled)
            dc::dispatch_kernel<MOE_F32, true><<<grid, dc::THREADS, 0, st>>>(xs, slot, gate, (int)T, k, vpr, R, xe, status_ptr(), row_gate);
        else
            dc::dispatch_kernel<MOE_F32, false><<<grid, dc::THREADS, 0, st>>>(xs, slot, gate, (int)T, k, vpr, R, xe, status_ptr(), row_gate);
    }
    return launch_status();
}

extern "C" int moe_dispatch(const void* x, const int32_t* slot, const float* gate, int64_t T,
                            int64_t d, int k, int dtype, void* Xe, void* stream) {
    return dispatch_impl(x, slot, gate, gate != nullptr, T, d, k, dtype, Xe, nullptr, stream);
}

extern "C" int moe_dispatch_gate(const void* x, const int32_t* slot, const float* gate, int64_t T,
                                 int64_t d, int k, int dtype, void* Xe, float* row_gate,
                                 void* stream) {
    if (T > 0 && (!gate || !row_gate)) return MOE_ERR_INVALID;
    return dispatch_impl(x, slot, gate, false, T, d, k, dtype, Xe, row_gate, stream);
}

extern "C" int moe_combine(const void* Ye, const int32_t* slot, const float* gate, int64_t T,
                           int64_t d, int k, int dtype, void* out, void* stream) {
    if (T < 0 || d <= 0 || k < 1 || k > MOE_MAX_TOPK) return MOE_ERR_INVALID;
    if (dtype != MOE_F32 && dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
    const int es = dtype == MOE_F32 ? 4 : 2;
    if ((d * es) % 16 != 0) return MOE_ERR_UNSUPPORTED;
    if (T == 0) return MOE_OK;
    if (!Ye || !slot || !out || !aligned16(Ye) || !aligned16(out)) return MOE_ERR_INVALID;
    if (T * k > INT32_MAX) return MOE_ERR_UNSUPPORTED;
    if (check_only()) return MOE_OK;
    const int vpr = (int)(d * es / 16);
    const int64_t R = T * k;
    cudaStream_t st = as_stream(stream);
    const int grid = dc::grid_for(T);
    const uint4* ye = static_cast<const uint4*>(Ye);
    uint4* o = static_cast<uint4*>(out);
    if (dtype == MOE_BF16) {
        if (gate)
            dc::combine_kernel<MOE_BF16, false><<<grid, dc::THREADS, 0, st>>>(ye, slot, gate, (int)T, k, vpr, R, o, status_ptr());
        else
            dc::combine_kernel<MOE_BF16, true><<<grid, dc::THREADS, 0, st>>>(ye, slot, gate, (int)T, k, vpr, R, o, status_ptr());
    } else {
        if (gate)
            dc::combine_kernel<MOE_F32, false><<<grid, dc::THREADS, 0, st>>>(ye, slot, gate, (int)T, k, vpr, R, o, status_ptr());
        else
            dc::combine_kernel<MOE_F32, true><<<grid, dc::THREADS, 0, st>>>(ye, slot, gate, (int)T, k, vpr, R, o, status_ptr());
    }
    return launch_status();
}

extern "C" int moe_row_token(const int32_t* slot, int64_t T, int k, int32_t* row_token,
                             void* stream) {
    if (T < 0 || k < 1 || k > MOE_MAX_TOPK) return MOE_ERR_INVALID;
    if (T == 0) return MOE_OK;
    if (!slot || !row_token) return MOE_ERR_INVALID;
    if (T * k > INT32_MAX) return MOE_ERR_UNSUPPORTED;
    if (check_only()) return MOE_OK;
    const int64_t n = T * k;
    int64_t g = (n + dc::THREADS - 1) / dc::THREADS;
    const int64_t cap = (int64_t)num_sms() * 8;
    if (g > cap) g = cap;
    dc::row_token_kernel<<<(int)g, dc::THREADS, 0, as_stream(stream)>>>(slot, n, k, n, row_token,
                                                                        status_ptr());
    return launch_status();
}
