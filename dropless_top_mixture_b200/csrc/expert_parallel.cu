// Expert parallelism over G ranks: row-wise dispatch into the owning rank's
// expert buffer and the gather back, with no separate permutation.
//
// "olmoforge" README, capability table: row-wise expert parallelism writes
// each token row straight into the input buffer of its expert, wherever that
// expert lives; "专家池 8→128 只慢 5%…" (Olmo-core 3, 关键数字): experts are
// spread over the GPUs and tokens travel to them. Rank r owns the El = E / G
// experts r El .. (r + 1) El - 1. After every rank's per-expert counts are
// gathered into C [G, E] (C[s][e] = rows rank s routes to expert e), every
// rank knows the layout of every receive buffer: rank r keeps the rows of
// its experts expert-major, and within an expert the rows of rank 0, then
// rank 1, ... in each sender's own (token-major) order. So a sender can
// write each of its (token, choice) rows straight to its final row in the
// owner's buffer:
//   dst_row(t, j) = recv_base_r(e) + sum_{s < me} C[s][e] + (slot[t,j] - offsets[e])
// with e = idx[t,j], r = e / El, recv_base_r(e) = rows of r's experts below e.
// The receive buffer is then the expert-sorted input of rank r's grouped
// GEMMs (offsets = recv_offsets), and the combine gathers each row's output
// back from the owner's output buffer at the same row.
//
// The buffers of all ranks are reached through a device table of G
// pointers: on a multi-GPU node the peers' buffers mapped into this process
// (loads and stores over NVLink); on one GPU, G buffer sets of one device.
#include "common.cuh"

namespace moe {
namespace ep {

constexpr int THREADS = 256;
constexpr int PLAN_THREADS = MOE_MAX_EXPERTS;
constexpr int MAX_RANKS = 64;

// base_me[e] = this rank's first row in expert e's segment of the owner's
// receive buffer; recv_offsets[0..El] = this rank's receive buffer offsets by
// local expert. One CTA of MOE_MAX_EXPERTS threads, thread e = expert e.
__global__ void __launch_bounds__(PLAN_THREADS)
    plan_base_kernel(const int32_t* __restrict__ C, int G, int E, int me,
                     int32_t* __restrict__ base_me, int32_t* __restrict__ recv_offsets,
                     int* status) {
    __shared__ int s_scan[PLAN_THREADS + 1];
    __shared__ int s_warp[PLAN_THREADS / 32];
    const int e = threadIdx.x, lane = e & 31, w = e >> 5;
    const int El = E / G;
    int tot = 0, below = 0;
    bool bad = false;
    if (e < E) {
        for (int s = 0; s < G; ++s) {
            const int c = C[(size_t)s * E + e];
            if (c < 0) bad = true;
            tot += c;
            if (s < me) below += c;
        }
    }
    if (bad) set_status(status, MOE_DEVERR_BAD_INDEX);
    // exclusive scan of tot over all experts (warp scans, then the warps')
    int wt;
    const int ex = warp_exclusive_scan(tot, &wt);
    if (lane == 0) s_warp[w] = wt;
    __syncthreads();
    if (w == 0) {
        const int v = lane < PLAN_THREADS / 32 ? s_warp[lane] : 0;
        int tt;
        const int e2 = warp_exclusive_scan(v, &tt);
        if (lane < PLAN_THREADS / 32) s_warp[lane] = e2;
    }
    __syncthreads();
    const int scan = ex + s_warp[w];
    s_scan[e] = scan;
    if (e == E - 1) s_scan[E] = scan + tot;
    __syncthreads();
    if (e < E) {
        const int r = e / El;
        const int seg = scan - s_scan[r * El];  // rows of r's experts below e
        base_me[e] = seg + below;
        if (r == me) recv_offsets[e - r * El] = seg;
    }
    if (e == 0) recv_offsets[El] = s_scan[(me + 1) * El] - s_scan[me * El];
}

// dst_rank, dst_row of every (token, choice) of this rank
__global__ void __launch_bounds__(THREADS)
    plan_rows_kernel(const int32_t* __restrict__ idx, const int32_t* __restrict__ slot,
                     const int32_t* __restrict__ offsets, const int32_t* __restrict__ base_me,
                     int64_t n, int E, int El, int32_t* __restrict__ dst_rank,
                     int32_t* __restrict__ dst_row, int* status) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int e = idx[i];
        if (e < 0 || e >= E) {
            set_status(status, MOE_DEVERR_BAD_INDEX);
            dst_rank[i] = -1;
            dst_row[i] = -1;
            continue;
        }
        dst_rank[i] = e / El;
        dst_row[i] = base_me[e] + (slot[i] - offsets[e]);
    }
}

// recv_bufs[dst_rank[t,j]][dst_row[t,j], :] = x[t, :]; a CTA reads x[t] once
// and writes its k copies in 16-byte vectors
__global__ void __launch_bounds__(THREADS)
    dispatch_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ dst_rank,
                    const int32_t* __restrict__ dst_row, int T, int k, int vpr, int G,
                    int64_t rows_max, uint4* const* __restrict__ bufs, int* status) {
    __shared__ uint4* s_dst[MOE_MAX_TOPK];
    for (int t = blockIdx.x; t < T; t += gridDim.x) {
        __syncthreads();
        if (threadIdx.x < k) {
            const int r = dst_rank[(size_t)t * k + threadIdx.x];
            const int row = dst_row[(size_t)t * k + threadIdx.x];
            uint4* p = nullptr;
            if (r >= 0 && r < G && row >= 0 && row < rows_max) p = bufs[r];
            if (reinterpret_cast<uintptr_t>(p) & 15u) p = nullptr;  // rows are 16-byte vectors
            if (p == nullptr) set_status(status, MOE_DEVERR_BAD_INDEX);
            s_dst[threadIdx.x] = p ? p + (size_t)row * vpr : nullptr;
        }
        __syncthreads();
        const uint4* src = x + (size_t)t * vpr;
        for (int v = threadIdx.x; v < vpr; v += THREADS) {
            const uint4 val = __ldcs(src + v);
            for (int j = 0; j < k; ++j) {
                uint4* dst = s_dst[j];
                if (dst) dst[v] = val;
            }
        }
    }
}

// out[t] = sum_j gate[t,j] * ye_bufs[dst_rank[t,j]][dst_row[t,j]], fp32 fused
// multiply-add in ascending j (no atomics, deterministic)
template <int DT>
__global__ void __launch_bounds__(THREADS)
    combine_kernel(const uint4* const* __restrict__ bufs, const int32_t* __restrict__ dst_rank,
                   const int32_t* __restrict__ dst_row, const float* __restrict__ gate, int T,
                   int k, int vpr, int G, int64_t rows_max, uint4* __restrict__ out,
                   int* status) {
    constexpr int N = DT == MOE_F32 ? 4 : 8;
    __shared__ const uint4* s_src[MOE_MAX_TOPK];
    __shared__ float s_gate[MOE_MAX_TOPK];
    for (int t = blockIdx.x; t < T; t += gridDim.x) {
        __syncthreads();
        if (threadIdx.x < k) {
            const int r = dst_rank[(size_t)t * k + threadIdx.x];
            const int row = dst_row[(size_t)t * k + threadIdx.x];
            const uint4* p = nullptr;
            if (r >= 0 && r < G && row >= 0 && row < rows_max) p = bufs[r];
            if (reinterpret_cast<uintptr_t>(p) & 15u) p = nullptr;  // rows are 16-byte vectors
            if (p == nullptr) set_status(status, MOE_DEVERR_BAD_INDEX);
            s_src[threadIdx.x] = p ? p + (size_t)row * vpr : nullptr;
            s_gate[threadIdx.x] = gate[(size_t)t * k + threadIdx.x];
        }
        __syncthreads();
        for (int v = threadIdx.x; v < vpr; v += THREADS) {
            float acc[N];
#pragma unroll
            for (int q = 0; q < N; ++q) acc[q] = 0.f;
            for (int j = 0; j < k; ++j) {
                const uint4* src = s_src[j];
                if (!src) continue;
                const uint4 u = __ldcs(src + v);
                float f[N];
                if (DT == MOE_F32) {
                    f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y);
                    f[2] = __uint_as_float(u.z); f[3] = __uint_as_float(u.w);
                } else {
                    unpack8(u, f);
                }
                const float g = s_gate[j];
#pragma unroll
                for (int q = 0; q < N; ++q) acc[q] = fmaf(g, f[q], acc[q]);
            }
            uint4 o;
            if (DT == MOE_F32)
                o = make_uint4(__float_as_uint(acc[0]), __float_as_uint(acc[1]),
                               __float_as_uint(acc[2]), __float_as_uint(acc[3]));
            else
                o = pack8(acc);
            out[(size_t)t * vpr + v] = o;
        }
    }
}

inline int grid_for(int64_t n) {
    const int64_t cap = (int64_t)num_sms() * 8;
    return (int)(n < cap ? (n > 0 ? n : 1) : cap);
}

}  // namespace ep
}  // namespace moe

using namespace moe;

extern "C" size_t moe_ep_workspace_size(int64_t E) {
    if (E < 1 || E > MOE_MAX_EXPERTS) return 0;
    return sizeof(int32_t) * (size_t)E;
}

extern "C" int moe_ep_plan(const int32_t* counts_all, int G, int me, const int32_t* idx,
                           const int32_t* slot, const int32_t* offsets, int64_t T, int64_t E,
                           int k, int32_t* dst_rank, int32_t* dst_row, int32_t* recv_offsets,
                           void* workspace, size_t workspace_bytes, void* stream) {
    if (G < 1 || G > ep::MAX_RANKS || me < 0 || me >= G) return MOE_ERR_INVALID;
    if (E < 1 || E > MOE_MAX_EXPERTS || E % G != 0) return MOE_ERR_INVALID;
    if (T < 0 || k < 1 || k > MOE_MAX_TOPK || k > E) return MOE_ERR_INVALID;
    if (T * k > INT32_MAX) return MOE_ERR_UNSUPPORTED;
    if (!counts_all || !recv_offsets || !workspace ||
        workspace_bytes < moe_ep_workspace_size(E))
        return MOE_ERR_INVALID;
    if (T > 0 && (!idx || !slot || !offsets || !dst_rank || !dst_row)) return MOE_ERR_INVALID;
    if (check_only()) return MOE_OK;
    cudaStream_t st = as_stream(stream);
    int32_t* base_me = static_cast<int32_t*>(workspace);
    ep::plan_base_kernel<<<1, ep::PLAN_THREADS, 0, st>>>(counts_all, G, (int)E, me, base_me,
                                                          recv_offsets, status_ptr());
    const int64_t n = T * k;
    if (n > 0) {
        const int g = ep::grid_for((n + ep::THREADS - 1) / ep::THREADS);
        ep::plan_rows_kernel<<<g, ep::THREADS, 0, st>>>(idx, slot, offsets, base_me, n, (int)E,
                                                        (int)(E / G), dst_rank, dst_row,
                                                        status_ptr());
    }
    return launch_status();
}

extern "C" int moe_dispatch_ep(const void* x, const int32_t* dst_rank, const int32_t* dst_row,
                               int64_t T, int64_t d, int k, int dtype, void* const* recv_bufs,
                               int G, int64_t rows_max, void* stream) {
    if (T < 0 || d <= 0 || k < 1 || k > MOE_MAX_TOPK || G < 1 || G > ep::MAX_RANKS ||
        rows_max < 0)
        return MOE_ERR_INVALID;
    if (dtype != MOE_F32 && dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
    const int es = dtype == MOE_F32 ? 4 : 2;
    if ((d * es) % 16 != 0) return MOE_ERR_UNSUPPORTED;
    if (T == 0) return MOE_OK;
    if (!x || !dst_rank || !dst_row || !recv_bufs || !aligned16(x)) return MOE_ERR_INVALID;
    if ((reinterpret_cast<uintptr_t>(recv_bufs) & 7u) != 0) return MOE_ERR_INVALID;
    if (T * k > INT32_MAX || rows_max > INT32_MAX) return MOE_ERR_UNSUPPORTED;
    if (check_only()) return MOE_OK;
    const int vpr = (int)(d * es / 16);
    ep::dispatch_kernel<<<ep::grid_for(T), ep::THREADS, 0, as_stream(stream)>>>(
        static_cast<const uint4*>(x), dst_rank, dst_row, (int)T, k, vpr, G, rows_max,
        reinterpret_cast<uint4* const*>(recv_bufs), status_ptr());
    return launch_status();
}

extern "C" int moe_combine_ep(const void* const* ye_bufs, const int32_t* dst_rank,
                              const int32_t* dst_row, const float* gate, int64_t T, int64_t d,
                              int k, int dtype, int G, int64_t rows_max, void* out,
                              void* stream) {
    if (T < 0 || d <= 0 || k < 1 || k > MOE_MAX_TOPK || G < 1 || G > ep::MAX_RANKS ||
        rows_max < 0)
        return MOE_ERR_INVALID;
    if (dtype != MOE_F32 && dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
    const int es = dtype == MOE_F32 ? 4 : 2;
    if ((d * es) % 16 != 0) return MOE_ERR_UNSUPPORTED;
    if (T == 0) return MOE_OK;
    if (!ye_bufs || !dst_rank || !dst_row || !gate || !out || !aligned16(out))
        return MOE_ERR_INVALID;
    if ((reinterpret_cast<uintptr_t>(ye_bufs) & 7u) != 0) return MOE_ERR_INVALID;
    if (T * k > INT32_MAX || rows_max > INT32_MAX) return MOE_ERR_UNSUPPORTED;
    if (check_only()) return MOE_OK;
    const int vpr = (int)(d * es / 16);
    const uint4* const* bufs = reinterpret_cast<const uint4* const*>(ye_bufs);
    if (dtype == MOE_BF16)
        ep::combine_kernel<MOE_BF16><<<ep::grid_for(T), ep::THREADS, 0, as_stream(stream)>>>(
            bufs, dst_rank, dst_row, gate, (int)T, k, vpr, G, rows_max, static_cast<uint4*>(out),
            status_ptr());
    else
        ep::combine_kernel<MOE_F32><<<ep::grid_for(T), ep::THREADS, 0, as_stream(stream)>>>(
            bufs, dst_rank, dst_row, gate, (int)T, k, vpr, G, rows_max, static_cast<uint4*>(out),
            status_ptr());
    return launch_status();
}
