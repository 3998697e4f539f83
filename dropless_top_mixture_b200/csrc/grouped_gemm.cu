// Grouped SwiGLU expert FFN on 5th-generation tensor cores (sm_100a).
//
// "Transformers 中的 OLMoE" (blog.gitcode.com) §3: every expert is a SwiGLU
// FFN, Ye = W2 (silu(W1 x) * W3 x), over the rows routed to it. "olmoforge"
// README, capability table (grouped GEMM): the many small per-expert matmuls
// run as one kernel. Here one persistent kernel walks a device-side tile
// table built from the routing offsets, so the host never learns the
// per-expert row counts.
//
// Two instantiations:
//   gate_up  H[r]  = silu(Xe[r] W1_eᵀ) * (Xe[r] W3_eᵀ)   B tile = [W1 rows; W3 rows]
//   down     Ye[r] = H[r] W2_eᵀ
//
// Tile = 128 rows (one expert's rows; the last tile of an expert overlaps the
// next expert's rows, which are computed and masked at the store) x MMA_N
// columns of B. One 128xMMA_Nx16 MMA per 32 bytes of K; K is staged 128
// bytes at a time by TMA with the 128-byte swizzle the MMA descriptors read.
//
// Gathered A (gate/up only). With GATHER the A operand is not a dispatched
// Xe buffer: row r of the tile is token row_token[r] of x, fetched by TMA
// tile::gather4 copies (four rows of one 128-byte K slab each; lane l of
// the producer warp fetches tile rows 4l..4l+3), so the dispatch copy of x
// into Xe and its re-read are never made ("olmoforge" README, row-wise
// expert parallelism: tokens go straight into the expert's input without a
// separate permutation). Measured on B200 this path is about 3x slower
// than dispatch + tiled TMA (a 512-byte gather per lane per slab cannot
// keep the tensor cores fed), so the layer does not use it.
//
// Warp roles (320 threads, one CTA per SM):
//   warp 0, lane 0   TMA producer over a STAGES-deep shared-memory ring
//                    (GATHER: all of warp 0)
//   warp 1           allocates TMEM; lane 0 issues tcgen05.mma
//   warps 2..9       epilogue: tcgen05.ld from TMEM (warp w reads lanes
//                    32*(w%4).., two warps per quarter split the columns),
//                    SwiGLU / conversion, row-masked stores
// The accumulator is double-buffered in TMEM (2 x MMA_N columns), so the
// epilogue of tile i overlaps the main loop of tile i+1.
//
// Every wait is bounded: after its time limit (2 s) the waiting thread sets
// MOE_DEVERR_TIMEOUT and an abort flag, all roles leave their loops, the MMA
// issuer drains its outstanding MMAs, the producer waits (again bounded) for
// its copies in flight, and TMEM is released before the CTA exits.
#include <type_traits>

#include "tc_sm100.cuh"

namespace moe {
namespace gg {

constexpr int BM = 128;
constexpr int STAGES = 4;
constexpr int EPI_WARPS = 8;  // two per TMEM lane quarter, one per column half
constexpr int THREADS = 64 + 32 * EPI_WARPS;
using namespace tc;

// ------------------------------------------------------------------ config

template <typename TIn, bool SWIGLU, int MMA_N_>
struct Cfg {
    static constexpr bool TF32 = std::is_same<TIn, float>::value;
    static constexpr int ES = (int)sizeof(TIn);
    static constexpr int BK = 128 / ES;           // elements per 128-byte K slab
    static constexpr int UMMA_K = 32 / ES;        // elements per MMA (32 bytes)
    static constexpr int KSTEPS = BK / UMMA_K;    // 4
    static constexpr int MMA_N = MMA_N_;          // B rows per tile
    static constexpr int OUT_N = SWIGLU ? MMA_N / 2 : MMA_N;
    static constexpr int A_BYTES = BM * 128;
    static constexpr int B_BYTES = MMA_N * 128;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int TMEM_COLS = 2 * MMA_N;   // two accumulator buffers
    static constexpr int TMEM_ALLOC = TMEM_COLS <= 256 ? 256 : 512;
    static constexpr int NUM_BARS = 2 * STAGES + 5;
    static constexpr int META_BYTES = NUM_BARS * 8 + 16 + 2 * 4 * (MOE_MAX_EXPERTS + 1);
    static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + META_BYTES;
    static constexpr uint32_t IDESC = make_idesc(TF32 ? 2u : 1u, BM, MMA_N);
    static_assert(OUT_N % 32 == 0, "epilogue works in 32-column chunks");
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
};

struct Tile {
    int e, row0, row_end, n0;
};

// Tile t -> (expert, rows, columns). Tiles are ordered expert by expert;
// inside an expert, n-block major and m-tile minor, so CTAs running at the
// same time share B (weight) tiles and A row blocks through L2.
__device__ __forceinline__ Tile decode_tile(int t, int NB, int E, int out_n, const int* s_toff,
                                            const int* s_off) {
    const int q = t / NB;
    int lo = 0, hi = E - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_toff[mid] <= q) lo = mid;
        else hi = mid - 1;
    }
    Tile tl;
    tl.e = lo;
    const int Me = s_toff[lo + 1] - s_toff[lo];
    const int l = t - s_toff[lo] * NB;
    const int nb = l / Me, m = l - nb * Me;
    tl.row0 = s_off[lo] + m * BM;
    tl.row_end = s_off[lo + 1];
    tl.n0 = nb * out_n;
    return tl;
}

template <typename TOut>
struct Store32;

template <>
struct Store32<__nv_bfloat16> {
    __device__ static void run(__nv_bfloat16* dst, const float* v) {
        uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
        for (int i = 0; i < 4; ++i) d[i] = pack8(v + 8 * i);
    }
};

template <>
struct Store32<float> {
    __device__ static void run(float* dst, const float* v) {
        float4* d = reinterpret_cast<float4*>(dst);
#pragma unroll
        for (int i = 0; i < 8; ++i) d[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
    }
};

__device__ __forceinline__ float silu_mul(float g, float u) { return g / (1.0f + __expf(-g)) * u; }

template <typename TIn, bool SWIGLU, int MMA_N, bool GATHER = false>
__global__ void __launch_bounds__(THREADS, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB0,
                        const __grid_constant__ CUtensorMap tmB1,
                        const int32_t* __restrict__ offsets, int E, int R, int K, int N,
                        TIn* __restrict__ out, int64_t ldo, TIn* __restrict__ save_a,
                        TIn* __restrict__ save_b, int* status,
                        const int32_t* __restrict__ row_token, int x_rows, int b_mode,
                        const float* __restrict__ row_gate) {
    using C = Cfg<TIn, SWIGLU, MMA_N>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* meta = smem + STAGES * C::STAGE_BYTES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(meta);
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(meta + C::NUM_BARS * 8);
    volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
    int* s_bad = reinterpret_cast<int*>(s_tmem + 2);
    int* s_off = reinterpret_cast<int*>(meta + C::NUM_BARS * 8 + 16);
    int* s_toff = s_off + (MOE_MAX_EXPERTS + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint64_t wl = wait_limit();  // the pipeline waits' time limit, read once

    // --- device-side tile table from the routing offsets (validated) -------
    for (int e = tid; e <= E; e += THREADS) s_off[e] = offsets[e];
    __syncthreads();
    if (warp == 0) {
        int carry = 0;
        bool bad = false;
        for (int base = 0; base < E; base += 32) {
            const int e = base + lane;
            int m = 0;
            if (e < E) {
                const int cnt = s_off[e + 1] - s_off[e];
                if (cnt < 0) bad = true;
                else m = (cnt + BM - 1) / BM;
            }
            int tot;
            const int ex = warp_exclusive_scan(m, &tot);
            if (e < E) s_toff[e] = carry + ex;
            carry += tot;
        }
        bad = __any_sync(0xffffffffu, bad) || s_off[0] != 0 || s_off[E] != R;
        if (lane == 0) {
            s_toff[E] = carry;
            *s_bad = bad ? 1 : 0;
        }
    }
    __syncthreads();
    if (*s_bad) {
        if (tid == 0 && blockIdx.x == 0) set_status(status, MOE_DEVERR_BAD_OFFSETS);
        return;
    }
    const int NB = N / C::OUT_N;
    const int total = s_toff[E] * NB;
    if ((int)blockIdx.x >= total) return;
    const int KB = K / C::BK;

    uint64_t* full = bars;
    uint64_t* empty = bars + STAGES;
    uint64_t* tfull = bars + 2 * STAGES;
    uint64_t* tempty = bars + 2 * STAGES + 2;
    uint64_t* drain = bars + 2 * STAGES + 4;

    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(smem_u32(full + s), 1);
            mbar_init(smem_u32(empty + s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(tfull + b), 1);
            mbar_init(smem_u32(tempty + b), EPI_WARPS);
        }
        mbar_init(smem_u32(drain), 1);
        *s_abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        prefetch_map(&tmA);
        prefetch_map(&tmB0);
        if (SWIGLU) prefetch_map(&tmB1);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(s_tmem), C::TMEM_ALLOC);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *s_tmem;

    if (GATHER && warp == 0) {
        // ------------------------------------------------ TMA producer, A
        // rows gathered from x by row_token (whole warp): lane l fetches tile
        // rows 4l..4l+3 of each K slab with one tile::gather4 copy
        int stage = 0;
        uint32_t phase = 0;
        uint32_t issued_mask = 0, issued_parity = 0;
        bool ok = true;
        // this lane's four token rows of the next tile, loaded one tile ahead
        // so their latency hides behind the current tile's copies; rows past
        // R (the last tile's overhang) fetch token 0, computed and masked;
        // a token outside [0, x_rows) is flagged and read as token 0
        int nxt[4];
        auto load_rows = [&](int t) {
            const Tile tn = decode_tile(t, NB, E, C::OUT_N, s_toff, s_off);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int r = tn.row0 + 4 * lane + j;
                int tk = r < R ? __ldg(row_token + r) : 0;
                if ((unsigned)tk >= (unsigned)x_rows) {
                    set_status(status, MOE_DEVERR_BAD_INDEX);
                    tk = 0;
                }
                nxt[j] = tk;
            }
        };
        load_rows(blockIdx.x);
        for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
            const Tile tl = decode_tile(t, NB, E, C::OUT_N, s_toff, s_off);
            const int tok[4] = {nxt[0], nxt[1], nxt[2], nxt[3]};
            if (t + (int)gridDim.x < total) load_rows(t + (int)gridDim.x);
            for (int kb = 0; kb < KB; ++kb) {
                bool w = true;
                if (lane == 0)
                    w = mbar_wait(smem_u32(empty + stage), phase ^ 1u, s_abort, status,
                                  wl);
                if (!__shfl_sync(0xffffffffu, w ? 1 : 0, 0)) {
                    ok = false;
                    break;
                }
                const uint32_t fb = smem_u32(full + stage);
                const uint32_t sa = smem_u32(smem + stage * C::STAGE_BYTES);
                const uint32_t sb = sa + C::A_BYTES;
                if (lane == 0) {
                    mbar_expect_tx(fb, C::STAGE_BYTES);
                    if (b_mode) {
                        tma_load_4d(sb, &tmB0, fb, kb * C::BK, tl.n0, 0, tl.e);
                    } else {
                        tma_load_3d(sb, &tmB0, fb, kb * C::BK, tl.n0, tl.e);
                        tma_load_3d(sb + C::B_BYTES / 2, &tmB1, fb, kb * C::BK, tl.n0, tl.e);
                    }
                    issued_mask |= 1u << stage;
                    issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
                }
                __syncwarp();
                tma_gather4(sa + (uint32_t)lane * 512u, &tmA, fb, kb * C::BK, tok[0], tok[1],
                            tok[2], tok[3]);
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        if (!ok && lane == 0) {
            for (int s = 0; s < STAGES; ++s)
                if ((issued_mask >> s) & 1u) {
                    volatile int no_abort = 0;
                    mbar_wait(smem_u32(full + s), (issued_parity >> s) & 1u, &no_abort, nullptr,
                              DRAIN_LIMIT_NS);
                }
        }
        __syncwarp();
    } else if (warp == 0 && lane == 0) {
        // ------------------------------------------------ TMA producer
        int stage = 0;
        uint32_t phase = 0;
        uint32_t issued_mask = 0, issued_parity = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
            const Tile tl = decode_tile(t, NB, E, C::OUT_N, s_toff, s_off);
            for (int kb = 0; kb < KB; ++kb) {
                if (!mbar_wait(smem_u32(empty + stage), phase ^ 1u, s_abort, status, wl)) {
                    ok = false;
                    break;
                }
                const uint32_t fb = smem_u32(full + stage);
                const uint32_t sa = smem_u32(smem + stage * C::STAGE_BYTES);
                const uint32_t sb = sa + C::A_BYTES;
                mbar_expect_tx(fb, C::STAGE_BYTES);
                tma_load_2d(sa, &tmA, fb, kb * C::BK, tl.row0);
                if (SWIGLU && b_mode) {
                    // W1 and W3 blocks in one copy (a map with both tensors
                    // as its third dimension)
                    tma_load_4d(sb, &tmB0, fb, kb * C::BK, tl.n0, 0, tl.e);
                } else if (SWIGLU) {
                    tma_load_3d(sb, &tmB0, fb, kb * C::BK, tl.n0, tl.e);
                    tma_load_3d(sb + C::B_BYTES / 2, &tmB1, fb, kb * C::BK, tl.n0, tl.e);
                } else {
                    tma_load_3d(sb, &tmB0, fb, kb * C::BK, tl.n0, tl.e);
                }
                issued_mask |= 1u << stage;
                issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        if (!ok) {
            // wait (bounded) for the copies this thread put in flight
            for (int s = 0; s < STAGES; ++s)
                if ((issued_mask >> s) & 1u) {
                    volatile int no_abort = 0;
                    mbar_wait(smem_u32(full + s), (issued_parity >> s) & 1u, &no_abort, nullptr,
                              DRAIN_LIMIT_NS);
                }
        }
    } else if (warp == 1 && lane == 0) {
        // ------------------------------------------------ MMA issuer
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        int i = 0;
        for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++i) {
            const int buf = i & 1;
            const uint32_t tp = (uint32_t)(i >> 1) & 1u;
            if (!mbar_wait(smem_u32(tempty + buf), tp ^ 1u, s_abort, status, wl)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t dt = tmem_base + (uint32_t)(buf * MMA_N);
            for (int kb = 0; kb < KB; ++kb) {
                if (!mbar_wait(smem_u32(full + stage), phase, s_abort, status, wl)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t sa = smem_u32(smem + stage * C::STAGE_BYTES);
                const uint64_t ad = sw128_desc(sa);
                const uint64_t bd = sw128_desc(sa + C::A_BYTES);
#pragma unroll
                for (int ks = 0; ks < C::KSTEPS; ++ks)
                    tc_mma<C::TF32>(dt, ad + 2 * ks, bd + 2 * ks, C::IDESC, (kb | ks) != 0);
                tc_commit(smem_u32(empty + stage));
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (ok) tc_commit(smem_u32(tfull + buf));
        }
        if (!ok) {
            // make sure every MMA this thread issued has finished with TMEM
            tc_commit(smem_u32(drain));
            volatile int no_abort = 0;
            mbar_wait(smem_u32(drain), 0, &no_abort, nullptr, DRAIN_LIMIT_NS);
        }
    } else if (warp >= 2) {
        // ------------------------------------------------ epilogue
        const int q = warp & 3;  // TMEM lane quarter this warp may access
        const int c_lo = ((warp - 2) >> 2) * (C::OUT_N / 64);  // this warp's half of the
        const int c_hi = c_lo + C::OUT_N / 64;                  // 32-column chunks
        const int r_in_tile = q * 32 + lane;
        // accumulator columns of the gate and up halves (b_mode 2: the
        // fused copy puts W3's block first)
        const int gcol = b_mode == 2 ? C::OUT_N : 0;
        const int ucol = b_mode == 2 ? 0 : C::OUT_N;
        int i = 0;
        for (int t = blockIdx.x; t < total; t += gridDim.x, ++i) {
            const Tile tl = decode_tile(t, NB, E, C::OUT_N, s_toff, s_off);
            const int buf = i & 1;
            const uint32_t tp = (uint32_t)(i >> 1) & 1u;
            if (!mbar_wait(smem_u32(tfull + buf), tp, s_abort, status, wl)) break;
            tc_fence_after();
            const uint32_t ta = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * MMA_N);
            const int grow = tl.row0 + r_in_tile;
            const bool valid = grow < tl.row_end;
            TIn* orow = out + (size_t)(valid ? grow : 0) * ldo + tl.n0;
            // down with gates: the row's gate scales its fp32 sums
            const float g = (!SWIGLU && row_gate != nullptr && valid) ? __ldg(row_gate + grow) : 1.f;
#pragma unroll 1
            for (int c = c_lo; c < c_hi; ++c) {
                uint32_t a[32];
                float v[32];
                tmem_ld32(ta + (SWIGLU ? gcol : 0) + c * 32, a);
                if constexpr (SWIGLU) {
                    uint32_t b[32];
                    tmem_ld32(ta + ucol + c * 32, b);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        v[j] = silu_mul(__uint_as_float(a[j]), __uint_as_float(b[j]));
                    if (save_a != nullptr && valid) {
                        // pre-activations kept for the backward pass
                        const size_t off = (size_t)grow * ldo + tl.n0 + c * 32;
                        Store32<TIn>::run(save_a + off, reinterpret_cast<const float*>(a));
                        Store32<TIn>::run(save_b + off, reinterpret_cast<const float*>(b));
                    }
                } else {
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j) v[j] = g * __uint_as_float(a[j]);
                }
                if (valid) Store32<TIn>::run(orow + c * 32, v);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(tempty + buf));
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) {
        __syncwarp();
        tmem_dealloc(tmem_base, C::TMEM_ALLOC);
    }
}

// ------------------------------------------------------------------ host

template <typename TIn, bool SWIGLU, int MMA_N, bool GATHER = false>
static int launch(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                  const int32_t* offsets, int64_t E, int64_t R, int64_t K, int64_t N, void* out,
                  int64_t ldo, cudaStream_t st, void* save_a = nullptr, void* save_b = nullptr,
                  const int32_t* row_token = nullptr, int64_t x_rows = 0, int b_mode = 0,
                  const float* row_gate = nullptr) {
    using C = Cfg<TIn, SWIGLU, MMA_N>;
    auto kern = grouped_gemm_kernel<TIn, SWIGLU, MMA_N, GATHER>;
    if (check_only()) return MOE_OK;
    static bool attr_done[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_done[dev]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 C::SMEM_BYTES) != cudaSuccess)
            return MOE_ERR_CUDA;
        attr_done[dev] = true;
    }
    const int64_t max_tiles = (R / BM + E) * (N / C::OUT_N);
    const int64_t sms = num_sms();
    const int grid = (int)(max_tiles < sms ? max_tiles : sms);
    if (grid <= 0) return MOE_OK;
    kern<<<grid, THREADS, C::SMEM_BYTES, st>>>(a, b0, b1, offsets, (int)E, (int)R, (int)K, (int)N,
                                              static_cast<TIn*>(out), ldo, static_cast<TIn*>(save_a),
                                              static_cast<TIn*>(save_b), status_ptr(), row_token,
                                              (int)x_rows, b_mode, row_gate);
    return launch_status();
}

// ---------------------------------------------------------------- CTA pairs
//
// The same computation on a 256-row x 256-column tile shared by a cluster of
// two CTAs (tcgen05 cta_group::2, M = 256). CTA r of the pair keeps rows
// row0 + 128 r .. + 127 of A and one half of the B tile in its own shared
// memory (SwiGLU: CTA 0 the W1 block, CTA 1 the W3 block; down: the two
// 128-row halves of the W2 block), so each CTA streams half the B bytes of
// the single-CTA tile for the same work. Both CTAs' TMA copies complete on
// the leader's (rank 0) stage barrier; the leader's elected thread issues
// the MMAs and its commits arrive on the stage-empty and accumulator-full
// barriers of both CTAs; each CTA drains its own 128 TMEM lanes and both
// arrive on the leader's accumulator-empty barrier. Cluster barriers bracket
// set-up and tear-down, so no CTA signals a barrier that is not live.
namespace pr {
constexpr int STAGES = 6;
constexpr int A_BYTES = BM * 128;   // this CTA's 128 rows of a 128-byte K slab
constexpr int BH_BYTES = 128 * 128; // this CTA's 128 of the 256 B rows
constexpr int STAGE_BYTES = A_BYTES + BH_BYTES;
constexpr int NUM_BARS = 2 * STAGES + 5;
constexpr int META_BYTES = NUM_BARS * 8 + 16 + 2 * 4 * (MOE_MAX_EXPERTS + 1);
constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + META_BYTES;
constexpr int PM = 2 * BM;          // rows per pair tile
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
}  // namespace pr

template <typename TIn, bool SWIGLU>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    grouped_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA,
                             const __grid_constant__ CUtensorMap tmB0,
                             const __grid_constant__ CUtensorMap tmB1,
                             const int32_t* __restrict__ offsets, int E, int R, int K, int N,
                             TIn* __restrict__ out, int64_t ldo, TIn* __restrict__ save_a,
                             TIn* __restrict__ save_b, int* status,
                             const float* __restrict__ row_gate) {
    constexpr bool TF32 = std::is_same<TIn, float>::value;
    constexpr int BK = 128 / (int)sizeof(TIn);
    constexpr int MMA_N = 256;
    constexpr int OUT_N = SWIGLU ? MMA_N / 2 : MMA_N;
    constexpr uint32_t IDESC = make_idesc(TF32 ? 2u : 1u, pr::PM, MMA_N);
    constexpr int STAGES = pr::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* meta = smem + STAGES * pr::STAGE_BYTES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(meta);
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(meta + pr::NUM_BARS * 8);
    volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
    int* s_bad = reinterpret_cast<int*>(s_tmem + 2);
    int* s_off = reinterpret_cast<int*>(meta + pr::NUM_BARS * 8 + 16);
    int* s_toff = s_off + (MOE_MAX_EXPERTS + 1);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint64_t wl = wait_limit();  // the pipeline waits' time limit, read once
    const uint32_t rank = cluster_ctarank();
    const int cid = (int)cluster_id_x(), ncl = (int)ncluster_x();

    // --- tile table of 256-row pair tiles from the routing offsets ---------
    for (int e = tid; e <= E; e += THREADS) s_off[e] = offsets[e];
    __syncthreads();
    if (warp == 0) {
        int carry = 0;
        bool bad = false;
        for (int base = 0; base < E; base += 32) {
            const int e = base + lane;
            int m = 0;
            if (e < E) {
                const int cnt = s_off[e + 1] - s_off[e];
                if (cnt < 0) bad = true;
                else m = (cnt + pr::PM - 1) / pr::PM;
            }
            int tot;
            const int ex = warp_exclusive_scan(m, &tot);
            if (e < E) s_toff[e] = carry + ex;
            carry += tot;
        }
        bad = __any_sync(0xffffffffu, bad) || s_off[0] != 0 || s_off[E] != R;
        if (lane == 0) {
            s_toff[E] = carry;
            *s_bad = bad ? 1 : 0;
        }
    }
    __syncthreads();
    // both CTAs of a pair see the same offsets, so they leave here together
    if (*s_bad) {
        if (tid == 0 && blockIdx.x == 0) set_status(status, MOE_DEVERR_BAD_OFFSETS);
        return;
    }
    const int NB = N / OUT_N;
    const int total = s_toff[E] * NB;
    if (cid >= total) return;
    const int KB = K / BK;

    uint64_t* full = bars;
    uint64_t* empty = bars + STAGES;
    uint64_t* tfull = bars + 2 * STAGES;
    uint64_t* tempty = bars + 2 * STAGES + 2;
    uint64_t* drain = bars + 2 * STAGES + 4;
    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(smem_u32(full + s), 1);
            mbar_init(smem_u32(empty + s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(tfull + b), 1);
            mbar_init(smem_u32(tempty + b), 2 * EPI_WARPS);
        }
        mbar_init(smem_u32(drain), 1);
        *s_abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        prefetch_map(&tmA);
        prefetch_map(&tmB0);
        if (SWIGLU) prefetch_map(&tmB1);
    }
    if (warp == 1) {
        tmem_alloc_pair(smem_u32(s_tmem), 512);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem_base = *s_tmem;
    const uint32_t leader_full = map_to_cta(smem_u32(full), 0);
    const uint32_t leader_tempty = map_to_cta(smem_u32(tempty), 0);

    if (warp == 0 && lane == 0) {
        // ------------------------------------------------ TMA producer (both CTAs)
        int stage = 0;
        uint32_t phase = 0, issued_mask = 0, issued_parity = 0;
        bool ok = true;
        for (int t = cid; t < total && ok; t += ncl) {
            const int q = t / NB;
            int lo = 0, hi = E - 1;
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (s_toff[mid] <= q) lo = mid;
                else hi = mid - 1;
            }
            const int Me = s_toff[lo + 1] - s_toff[lo];
            const int l = t - s_toff[lo] * NB;
            const int nb = l / Me, m = l - nb * Me;
            const int arow = s_off[lo] + m * pr::PM + (int)rank * BM;
            const int n0 = nb * OUT_N;
            for (int kb = 0; kb < KB; ++kb) {
                if (!mbar_wait(smem_u32(empty + stage), phase ^ 1u, s_abort, status, wl)) {
                    ok = false;
                    break;
                }
                const uint32_t fb = leader_full + (uint32_t)stage * 8u;
                if (rank == 0) mbar_expect_tx(smem_u32(full + stage), 2 * pr::STAGE_BYTES);
                const uint32_t sa = smem_u32(smem + stage * pr::STAGE_BYTES);
                tma_load_2d_pair(sa, &tmA, fb, kb * BK, arow);
                if (SWIGLU)
                    tma_load_3d_pair(sa + pr::A_BYTES, rank == 0 ? &tmB0 : &tmB1, fb, kb * BK, n0, lo);
                else
                    tma_load_3d_pair(sa + pr::A_BYTES, &tmB0, fb, kb * BK, n0 + (int)rank * 128, lo);
                issued_mask |= 1u << stage;
                issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        if (!ok) {
            // the leader's stage barriers count both CTAs' copies: wait there
            // (bounded); the partner gives its copies a bounded grace period
            if (rank == 0) {
                for (int s = 0; s < STAGES; ++s)
                    if ((issued_mask >> s) & 1u) {
                        volatile int no_abort = 0;
                        mbar_wait(smem_u32(full + s), (issued_parity >> s) & 1u, &no_abort, nullptr,
                                  DRAIN_LIMIT_NS);
                    }
            } else {
                const uint64_t t0 = global_timer_ns();
                while (global_timer_ns() - t0 < 1000000ull) {
                }
            }
        }
    } else if (warp == 1 && lane == 0 && rank == 0) {
        // ------------------------------------------------ MMA issuer (leader)
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        int i = 0;
        for (int t = cid; t < total && ok; t += ncl, ++i) {
            const int buf = i & 1;
            const uint32_t tp = (uint32_t)(i >> 1) & 1u;
            if (!mbar_wait(smem_u32(tempty + buf), tp ^ 1u, s_abort, status, wl)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t dt = tmem_base + (uint32_t)(buf * MMA_N);
            for (int kb = 0; kb < KB; ++kb) {
                if (!mbar_wait(smem_u32(full + stage), phase, s_abort, status, wl)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t sa = smem_u32(smem + stage * pr::STAGE_BYTES);
                const uint64_t ad = sw128_desc(sa);
                const uint64_t bd = sw128_desc(sa + pr::A_BYTES);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    tc_mma_pair<TF32>(dt, ad + 2 * ks, bd + 2 * ks, IDESC, (kb | ks) != 0);
                tc_commit_pair(smem_u32(empty + stage), 0x3);
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (ok) tc_commit_pair(smem_u32(tfull + buf), 0x3);
        }
        if (!ok) {
            tc_commit_pair(smem_u32(drain), 0x1);
            volatile int no_abort = 0;
            mbar_wait(smem_u32(drain), 0, &no_abort, nullptr, DRAIN_LIMIT_NS);
        }
    } else if (warp >= 2) {
        // ------------------------------------------------ epilogue (both CTAs)
        const int qd = warp & 3;
        const int c_lo = ((warp - 2) >> 2) * (OUT_N / 64);
        const int c_hi = c_lo + OUT_N / 64;
        const int r_in_tile = qd * 32 + lane;
        int i = 0;
        for (int t = cid; t < total; t += ncl, ++i) {
            const int q = t / NB;
            int lo = 0, hi = E - 1;
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (s_toff[mid] <= q) lo = mid;
                else hi = mid - 1;
            }
            const int Me = s_toff[lo + 1] - s_toff[lo];
            const int l = t - s_toff[lo] * NB;
            const int nb = l / Me, m = l - nb * Me;
            const int row_end = s_off[lo + 1];
            const int n0 = nb * OUT_N;
            const int buf = i & 1;
            const uint32_t tp = (uint32_t)(i >> 1) & 1u;
            if (!mbar_wait(smem_u32(tfull + buf), tp, s_abort, status, wl)) break;
            tc_fence_after();
            const uint32_t ta = tmem_base + ((uint32_t)(qd * 32) << 16) + (uint32_t)(buf * MMA_N);
            const int grow = s_off[lo] + m * pr::PM + (int)rank * BM + r_in_tile;
            const bool valid = grow < row_end;
            TIn* orow = out + (size_t)(valid ? grow : 0) * ldo + n0;
            const float g = (!SWIGLU && row_gate != nullptr && valid) ? __ldg(row_gate + grow) : 1.f;
#pragma unroll 1
            for (int c = c_lo; c < c_hi; ++c) {
                uint32_t a[32];
                float v[32];
                tmem_ld32(ta + c * 32, a);
                if constexpr (SWIGLU) {
                    uint32_t b[32];
                    tmem_ld32(ta + OUT_N + c * 32, b);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        v[j] = silu_mul(__uint_as_float(a[j]), __uint_as_float(b[j]));
                    if (save_a != nullptr && valid) {
                        const size_t off = (size_t)grow * ldo + n0 + c * 32;
                        Store32<TIn>::run(save_a + off, reinterpret_cast<const float*>(a));
                        Store32<TIn>::run(save_b + off, reinterpret_cast<const float*>(b));
                    }
                } else {
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j) v[j] = g * __uint_as_float(a[j]);
                }
                if (valid) Store32<TIn>::run(orow + c * 32, v);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(leader_tempty + (uint32_t)buf * 8u);
        }
    }

    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    if (warp == 1) {
        __syncwarp();
        tmem_dealloc_pair(tmem_base, 512);
    }
}

template <typename TIn, bool SWIGLU>
static int launch_pair(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                       const int32_t* offsets, int64_t E, int64_t R, int64_t K, int64_t N,
                       void* out, int64_t ldo, cudaStream_t st, void* save_a = nullptr,
                       void* save_b = nullptr, const float* row_gate = nullptr) {
    auto kern = grouped_gemm_pair_kernel<TIn, SWIGLU>;
    if (check_only()) return MOE_OK;
    static bool attr_done[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_done[dev]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 pr::SMEM_BYTES) != cudaSuccess)
            return MOE_ERR_CUDA;
        attr_done[dev] = true;
    }
    const int out_n = SWIGLU ? 128 : 256;
    const int64_t max_pairs = (R / pr::PM + E) * (N / out_n);
    const int64_t pairs = num_sms() / 2;
    const int npairs = (int)(max_pairs < pairs ? max_pairs : pairs);
    if (npairs <= 0) return MOE_OK;
    kern<<<2 * npairs, THREADS, pr::SMEM_BYTES, st>>>(a, b0, b1, offsets, (int)E, (int)R, (int)K,
                                                      (int)N, static_cast<TIn*>(out), ldo,
                                                      static_cast<TIn*>(save_a),
                                                      static_cast<TIn*>(save_b), status_ptr(),
                                                      row_gate);
    return launch_status();
}

// ------------------------------------------------------ token-column tiles
//
// The same products with the operands' roles swapped: the 256 MMA rows of a
// CTA pair are weight rows and its N columns are one expert's tokens, so a
// tile covers N = 16 .. 256 tokens in steps of 16 rather than 128 or 256
// rows. An expert of c rows is cut into chunks of 256 rows and a last chunk
// of the remaining rows rounded up to 16, so the MMAs compute at most 15
// masked rows per expert (experts of about 256 rows: 3% of the MMA work,
// against 20% for 128-row tiles).
//
// Each pipeline stage holds two 128-byte K slabs, and each CTA fetches it
// with two TMA copies (one of weights, one of tokens) of up to 32 KB: on
// B200 the copy engine's rate depends on the number of copies far more than
// on their size (two 16 KB copies per 32 KB stage stream about two thirds
// as fast as one 32 KB copy), so the weight and token boxes each span both
// slabs through a map whose last dimension steps 128 bytes along K.
//
// gate/up: a 5-D map over the W1 and W3 rows delivers, for each TMEM lane
// quarter q of CTA r, 16 rows of the first tensor and then the same 16
// features' rows of the second (features f0 + 64 r + 16 q ..), so lanes l
// and l + 16 of an epilogue warp hold the gate and up pre-activations of
// one feature and one shuffle pairs them for the SwiGLU; the pair covers 128
// features of H. down: CTA r holds 128 rows of W2 (output features
// f0 + 128 r ..); the pair covers 256. Tokens: CTA r copies rows
// row0 + r N/2 .. with the smallest box of 8 .. 128 rows that covers N/2
// (rows past the chunk are fetched and never multiplied). Accumulator column
// c is token row0 + c and TMEM lane i is feature i of the CTA's rows, so the
// epilogue writes each token's run of the quarter's features (32 or 64
// contiguous bytes). Tiles run expert by expert, feature block major and
// chunk minor, so the chunks that share a weight block run together.
namespace sw {
constexpr int STAGES = 3;
constexpr int SLABS = 2;                    // 128-byte K slabs per stage
constexpr int A_BYTES = SLABS * 128 * 128;  // 128 weight rows
constexpr int B_BYTES = SLABS * 128 * 128;  // up to 128 token rows (half of N = 256)
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int NUM_BARS = 2 * STAGES + 5;
constexpr int META_BYTES = NUM_BARS * 8 + 16 + 2 * 4 * (MOE_MAX_EXPERTS + 1);
constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + META_BYTES;
constexpr int NBOX = 5;                     // token boxes of 8, 16, 32, 64, 128 rows
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");

struct TokenMaps {
    CUtensorMap m[NBOX];
};

struct Chunk {
    int e, fb, row0, row_end, n;
};

// Tile t -> (expert, feature block, token chunk); s_toff is the prefix of
// the experts' chunk counts.
__device__ __forceinline__ Chunk decode(int t, int FB, int E, const int* s_toff, const int* s_off) {
    const int q = t / FB;
    int lo = 0, hi = E - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_toff[mid] <= q) lo = mid;
        else hi = mid - 1;
    }
    const int ch = s_toff[lo + 1] - s_toff[lo];
    const int l = t - s_toff[lo] * FB;
    const int fb = l / ch, j = l - fb * ch;
    Chunk c;
    c.e = lo;
    c.fb = fb;
    c.row0 = s_off[lo] + 256 * j;
    const int rows = min(256, s_off[lo + 1] - c.row0);
    c.row_end = c.row0 + rows;
    c.n = (rows + 15) & ~15;
    return c;
}

// smallest token box (index into TokenMaps) covering `half` rows
__device__ __forceinline__ int box_sel(int half) {
    return half <= 8 ? 0 : half <= 16 ? 1 : half <= 32 ? 2 : half <= 64 ? 3 : 4;
}

template <typename T>
__device__ __forceinline__ T to_out(float v);
template <>
__device__ __forceinline__ __nv_bfloat16 to_out<__nv_bfloat16>(float v) {
    return __float2bfloat16_rn(v);
}
template <>
__device__ __forceinline__ float to_out<float>(float v) {
    return v;
}
}  // namespace sw

template <typename TIn, bool SWIGLU>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    grouped_gemm_swap_kernel(const __grid_constant__ CUtensorMap tmW,
                             const __grid_constant__ sw::TokenMaps tmX,
                             const int32_t* __restrict__ offsets, int E, int R, int K, int NOUT,
                             int wpe, int second_is_gate, TIn* __restrict__ out, int64_t ldo,
                             TIn* __restrict__ save_a, TIn* __restrict__ save_b, int* status,
                             const float* __restrict__ row_gate) {
    constexpr bool TF32 = std::is_same<TIn, float>::value;
    constexpr int BK = 128 / (int)sizeof(TIn);
    constexpr uint32_t IDESC_M = make_idesc(TF32 ? 2u : 1u, 256, 0);  // N filled per tile
    constexpr int STAGES = sw::STAGES;
    constexpr int FEAT = SWIGLU ? 128 : 256;  // output features per pair tile
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* meta = smem + STAGES * sw::STAGE_BYTES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(meta);
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(meta + sw::NUM_BARS * 8);
    volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
    int* s_bad = reinterpret_cast<int*>(s_tmem + 2);
    int* s_off = reinterpret_cast<int*>(meta + sw::NUM_BARS * 8 + 16);
    int* s_toff = s_off + (MOE_MAX_EXPERTS + 1);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint64_t wl = wait_limit();  // the pipeline waits' time limit, read once
    const uint32_t rank = cluster_ctarank();
    const int cid = (int)cluster_id_x(), ncl = (int)ncluster_x();

    // --- chunk table from the routing offsets (validated) ------------------
    for (int e = tid; e <= E; e += THREADS) s_off[e] = offsets[e];
    __syncthreads();
    if (warp == 0) {
        int carry = 0;
        bool bad = false;
        for (int base = 0; base < E; base += 32) {
            const int e = base + lane;
            int ch = 0;
            if (e < E) {
                const int cnt = s_off[e + 1] - s_off[e];
                if (cnt < 0) bad = true;
                else ch = (cnt + 255) >> 8;
            }
            int tot;
            const int ex = warp_exclusive_scan(ch, &tot);
            if (e < E) s_toff[e] = carry + ex;
            carry += tot;
        }
        bad = __any_sync(0xffffffffu, bad) || s_off[0] != 0 || s_off[E] != R;
        if (lane == 0) {
            s_toff[E] = carry;
            *s_bad = bad ? 1 : 0;
        }
    }
    __syncthreads();
    // both CTAs of a pair see the same offsets, so they leave here together
    if (*s_bad) {
        if (tid == 0 && blockIdx.x == 0) set_status(status, MOE_DEVERR_BAD_OFFSETS);
        return;
    }
    const int FB = NOUT / FEAT;
    const int total = s_toff[E] * FB;
    if (cid >= total) return;
    const int KS = K / (sw::SLABS * BK);  // stages per tile

    uint64_t* full = bars;
    uint64_t* empty = bars + STAGES;
    uint64_t* tfull = bars + 2 * STAGES;
    uint64_t* tempty = bars + 2 * STAGES + 2;
    uint64_t* drain = bars + 2 * STAGES + 4;
    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(smem_u32(full + s), 1);
            mbar_init(smem_u32(empty + s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(tfull + b), 1);
            mbar_init(smem_u32(tempty + b), 2 * EPI_WARPS);
        }
        mbar_init(smem_u32(drain), 1);
        *s_abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        prefetch_map(&tmW);
        for (int b = 0; b < sw::NBOX; ++b) prefetch_map(&tmX.m[b]);
    }
    if (warp == 1) {
        tmem_alloc_pair(smem_u32(s_tmem), 512);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem_base = *s_tmem;
    const uint32_t leader_full = map_to_cta(smem_u32(full), 0);
    const uint32_t leader_tempty = map_to_cta(smem_u32(tempty), 0);

    if (warp == 0 && lane == 0) {
        // ------------------------------------------------ TMA producer (both CTAs)
        int stage = 0;
        uint32_t phase = 0, issued_mask = 0, issued_parity = 0;
        bool ok = true;
        for (int t = cid; t < total && ok; t += ncl) {
            const sw::Chunk c = sw::decode(t, FB, E, s_toff, s_off);
            const int half = c.n >> 1;  // token rows of this CTA (a multiple of 8)
            const int bs = sw::box_sel(half);
            const CUtensorMap* xm = &tmX.m[bs];
            const int brow = c.row0 + (int)rank * half;
            const uint32_t tx = 2u * (uint32_t)(sw::A_BYTES + (8 << bs) * 128 * sw::SLABS);
            const int wcoord = SWIGLU ? c.e * wpe + c.fb * 8 + 4 * (int)rank
                                      : c.e * wpe + c.fb * FEAT + 128 * (int)rank;
            for (int ks = 0; ks < KS; ++ks) {
                if (!mbar_wait(smem_u32(empty + stage), phase ^ 1u, s_abort, status, wl)) {
                    ok = false;
                    break;
                }
                const uint32_t fbar = leader_full + (uint32_t)stage * 8u;
                const uint32_t sa = smem_u32(smem + stage * sw::STAGE_BYTES);
                if (rank == 0) mbar_expect_tx(smem_u32(full + stage), tx);
                if (SWIGLU)
                    tma_load_5d_pair(sa, &tmW, fbar, 0, 0, 0, wcoord, sw::SLABS * ks);
                else
                    tma_load_3d_pair(sa, &tmW, fbar, 0, wcoord, sw::SLABS * ks);
                tma_load_3d_pair(sa + sw::A_BYTES, xm, fbar, 0, brow, sw::SLABS * ks);
                issued_mask |= 1u << stage;
                issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        if (!ok) {
            // the leader's stage barriers count both CTAs' copies: wait there
            // (bounded); the partner gives its copies a bounded grace period
            if (rank == 0) {
                for (int s = 0; s < STAGES; ++s)
                    if ((issued_mask >> s) & 1u) {
                        volatile int no_abort = 0;
                        mbar_wait(smem_u32(full + s), (issued_parity >> s) & 1u, &no_abort, nullptr,
                                  DRAIN_LIMIT_NS);
                    }
            } else {
                const uint64_t t0 = global_timer_ns();
                while (global_timer_ns() - t0 < 1000000ull) {
                }
            }
        }
    } else if (warp == 1 && lane == 0 && rank == 0) {
        // ------------------------------------------------ MMA issuer (leader)
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        int i = 0;
        for (int t = cid; t < total && ok; t += ncl, ++i) {
            const sw::Chunk c = sw::decode(t, FB, E, s_toff, s_off);
            const uint32_t idesc = IDESC_M | ((uint32_t)(c.n >> 3) << 17);
            const uint32_t bslab = (uint32_t)(8 << sw::box_sel(c.n >> 1)) * 128u;  // B slab stride
            const int buf = i & 1;
            const uint32_t tp = (uint32_t)(i >> 1) & 1u;
            if (!mbar_wait(smem_u32(tempty + buf), tp ^ 1u, s_abort, status, wl)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t dt = tmem_base + (uint32_t)(buf * 256);
            for (int ks = 0; ks < KS; ++ks) {
                if (!mbar_wait(smem_u32(full + stage), phase, s_abort, status, wl)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t sa = smem_u32(smem + stage * sw::STAGE_BYTES);
#pragma unroll
                for (int sl = 0; sl < sw::SLABS; ++sl) {
                    const uint64_t ad = sw128_desc(sa + (uint32_t)sl * (128u * 128u));
                    const uint64_t bd = sw128_desc(sa + sw::A_BYTES + (uint32_t)sl * bslab);
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        tc_mma_pair<TF32>(dt, ad + 2 * k, bd + 2 * k, idesc, (ks | sl | k) != 0);
                }
                tc_commit_pair(smem_u32(empty + stage), 0x3);
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (ok) tc_commit_pair(smem_u32(tfull + buf), 0x3);
        }
        if (!ok) {
            tc_commit_pair(smem_u32(drain), 0x1);
            volatile int no_abort = 0;
            mbar_wait(smem_u32(drain), 0, &no_abort, nullptr, DRAIN_LIMIT_NS);
        }
    } else if (warp >= 2) {
        // ------------------------------------------------ epilogue (both CTAs)
        // warp w reads TMEM lane quarter w % 4; the two warps of a quarter
        // take alternate 32-column (token) chunks
        const int qd = warp & 3;
        const int h = (warp - 2) >> 2;
        const bool lo = lane < 16;
        const bool holds_gate = lo != (second_is_gate != 0);
        int i = 0;
        for (int t = cid; t < total; t += ncl, ++i) {
            const sw::Chunk c = sw::decode(t, FB, E, s_toff, s_off);
            const int buf = i & 1;
            const uint32_t tp = (uint32_t)(i >> 1) & 1u;
            if (!mbar_wait(smem_u32(tfull + buf), tp, s_abort, status, wl)) break;
            tc_fence_after();
            const uint32_t ta = tmem_base + ((uint32_t)(qd * 32) << 16) + (uint32_t)(buf * 256);
            const int f = SWIGLU ? c.fb * FEAT + 64 * (int)rank + 16 * qd + (lane & 15)
                                 : c.fb * FEAT + 128 * (int)rank + 32 * qd + lane;
            const int nch = (c.n + 31) >> 5;
#pragma unroll 1
            for (int ck = h; ck < nch; ck += 2) {
                uint32_t a[32];
                tmem_ld32(ta + (uint32_t)(ck * 32), a);
                tmem_wait_ld();
                const int tok0 = c.row0 + ck * 32;
                if constexpr (SWIGLU) {
                    if (save_a != nullptr) {
                        // pre-activations kept for the backward pass
                        TIn* dst = holds_gate ? save_a : save_b;
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            if (tok0 + j < c.row_end)
                                dst[(size_t)(tok0 + j) * ldo + f] =
                                    sw::to_out<TIn>(__uint_as_float(a[j]));
                    }
                    // lane l < 16 finishes tokens 0..15 of the chunk with the
                    // values of lane l + 16, which finishes tokens 16..31
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const float mine_lo = __uint_as_float(a[j]);
                        const float mine_hi = __uint_as_float(a[16 + j]);
                        const float other =
                            __shfl_xor_sync(0xffffffffu, lo ? mine_hi : mine_lo, 16);
                        const float mine = lo ? mine_lo : mine_hi;
                        const float g = holds_gate ? mine : other;
                        const float u = holds_gate ? other : mine;
                        const int tok = tok0 + (lo ? 0 : 16) + j;
                        if (tok < c.row_end)
                            out[(size_t)tok * ldo + f] = sw::to_out<TIn>(silu_mul(g, u));
                    }
                } else {
                    // down with gates: column j is token row tok0 + j; lane j
                    // fetches its gate and the shuffle hands it to every lane
                    float gl = 1.f;
                    if (row_gate != nullptr && tok0 + lane < c.row_end) gl = __ldg(row_gate + tok0 + lane);
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const float gj = __shfl_sync(0xffffffffu, gl, j);
                        if (tok0 + j < c.row_end)
                            out[(size_t)(tok0 + j) * ldo + f] =
                                sw::to_out<TIn>(gj * __uint_as_float(a[j]));
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(leader_tempty + (uint32_t)buf * 8u);
        }
    }

    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    if (warp == 1) {
        __syncwarp();
        tmem_dealloc_pair(tmem_base, 512);
    }
}

// Token maps over X [R, K]: dims (128-byte slab, rows, slabs), boxes of
// 8 .. 128 rows spanning two slabs.
inline bool make_token_maps(sw::TokenMaps* tm, const void* X, CUtensorMapDataType dt, int es,
                            int64_t K, int64_t R) {
    const uint64_t bk = 128 / es;
    const uint64_t dims[3] = {bk, (uint64_t)R, (uint64_t)K / bk};
    const uint64_t strides[2] = {(uint64_t)K * es, 128};
    for (int b = 0; b < sw::NBOX; ++b) {
        const uint32_t box[3] = {(uint32_t)bk, 8u << b, (uint32_t)sw::SLABS};
        if (!make_map_nd(&tm->m[b], X, dt, 3, dims, strides, box)) return false;
    }
    return true;
}

// gate/up weight map: dims (slab, 16 rows, 2 tensors, 16-row groups, slabs)
// over the W1 and W3 rows, the lower address first; needs the expert stride
// to be a whole number of 16-row groups and the two tensors a multiple of 16
// bytes apart. *second_is_gate tells which tensor is first.
inline bool gate_up_map_fits(const void* W1, const void* W3, int64_t estride, int64_t E,
                             int64_t d, int es) {
    const int64_t diff = (int64_t)((const char*)W3 - (const char*)W1);
    const int64_t ad = diff < 0 ? -diff : diff;
    return ad > 0 && ad % 16 == 0 && ad < (int64_t(1) << 40) && (E == 1 || estride % (16 * d) == 0) &&
           (int64_t)d * es < (int64_t(1) << 40);
}
inline bool make_gate_up_map(CUtensorMap* m, const void* W1, const void* W3, CUtensorMapDataType dt,
                             int es, int64_t estride, int64_t E, int64_t d, int64_t F, int* wpe,
                             int* second_is_gate) {
    const bool w3_first = (const char*)W3 < (const char*)W1;
    const void* base = w3_first ? W3 : W1;
    const int64_t diff = w3_first ? (const char*)W1 - (const char*)W3 : (const char*)W3 - (const char*)W1;
    const int64_t gpe = E == 1 ? F / 16 : estride / (16 * d);
    const uint64_t bk = 128 / es;
    const uint64_t dims[5] = {bk, 16, 2, (uint64_t)((E - 1) * gpe + F / 16), (uint64_t)d / bk};
    const uint64_t strides[4] = {(uint64_t)d * es, (uint64_t)diff, (uint64_t)(16 * d * es), 128};
    const uint32_t box[5] = {(uint32_t)bk, 16, 2, 4, (uint32_t)sw::SLABS};
    *wpe = (int)gpe;
    *second_is_gate = w3_first ? 1 : 0;
    return make_map_nd(m, base, dt, 5, dims, strides, box);
}
// down weight map: dims (slab, rows of all experts, slabs) over W2 [E, d, F];
// needs the expert stride to be a whole number of rows.
inline bool down_map_fits(int64_t estride, int64_t E, int64_t F) {
    return E == 1 || estride % F == 0;
}
inline bool make_down_map(CUtensorMap* m, const void* W2, CUtensorMapDataType dt, int es,
                          int64_t estride, int64_t E, int64_t d, int64_t F, int* wpe) {
    const int64_t rpe = E == 1 ? d : estride / F;
    const uint64_t bk = 128 / es;
    const uint64_t dims[3] = {bk, (uint64_t)((E - 1) * rpe + d), (uint64_t)F / bk};
    const uint64_t strides[2] = {(uint64_t)F * es, 128};
    const uint32_t box[3] = {(uint32_t)bk, 128, (uint32_t)sw::SLABS};
    *wpe = (int)rpe;
    return make_map_nd(m, W2, dt, 3, dims, strides, box);
}

template <typename TIn, bool SWIGLU>
static int launch_swap(const CUtensorMap& w, const sw::TokenMaps& x, const int32_t* offsets,
                       int64_t E, int64_t R, int64_t K, int64_t NOUT, int wpe, int second_is_gate,
                       void* out, int64_t ldo, cudaStream_t st, void* save_a = nullptr,
                       void* save_b = nullptr, const float* row_gate = nullptr) {
    auto kern = grouped_gemm_swap_kernel<TIn, SWIGLU>;
    if (check_only()) return MOE_OK;
    static bool attr_done[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_done[dev]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 sw::SMEM_BYTES) != cudaSuccess)
            return MOE_ERR_CUDA;
        attr_done[dev] = true;
    }
    const int64_t feat = SWIGLU ? 128 : 256;
    const int64_t max_tiles = (R / 256 + E) * (NOUT / feat);
    const int64_t pairs = num_sms() / 2;
    const int npairs = (int)(max_tiles < pairs ? max_tiles : pairs);
    if (npairs <= 0) return MOE_OK;
    kern<<<2 * npairs, THREADS, sw::SMEM_BYTES, st>>>(
        w, x, offsets, (int)E, (int)R, (int)K, (int)NOUT, wpe, second_is_gate,
        static_cast<TIn*>(out), ldo, static_cast<TIn*>(save_a), static_cast<TIn*>(save_b),
        status_ptr(), row_gate);
    return launch_status();
}

// Measured on B200: the pair tile speeds up the down GEMM (olmoe-shaped layer
// 1071 -> 1143 TFLOP/s) but not gate/up, which already runs at the
// power-capped clock; with about 256 rows per expert the pair's second half
// computes many rows it then masks (128-expert sweep: slower). So it is
// used for the down GEMM when experts average at least 512 rows.
inline bool use_pair(int64_t R, int64_t E) { return R >= 512 * E; }

// Tile form: 0 = chosen by shape, 1 = row tiles, 2 = token-column tiles
// (where the weight strides allow them). Set by moe_debug_set_gemm_form.
inline int& gemm_form() {
    static int form = 0;
    return form;
}

// Measured on B200 (bf16, power-capped layer steps and isolated calls):
// token-column tiles run gate/up 8-12% and down up to 26% faster than row
// tiles when experts average 512 rows or more (OLMoE-shaped layer, 8 and 32
// experts of the sweep); at about 256 rows per expert (128-expert sweep) the
// last chunk of each expert streams a whole weight block for a few tokens
// and row tiles are about 4% faster; below that the two trade places from
// run to run. So: token columns from 512 rows per expert on.
inline bool use_swap(int64_t R, int64_t E) {
    const int f = gemm_form();
    if (f != 0) return f == 2;
    return R >= 512 * E;
}

// Row-tile gate/up B map: dims (slab, F rows, 2 tensors, E) over W1 and W3,
// the lower address first, so one copy fetches both 128-row blocks. Returns
// the mode for the kernel (1: W1 first, 2: W3 first) or 0 when the two
// tensors are not a multiple of 16 bytes apart (two maps then).
inline int make_w13_map(CUtensorMap* m, const void* W1, const void* W3, CUtensorMapDataType dt,
                        int es, int64_t estride, int64_t E, int64_t d, int64_t F) {
    const int64_t diff = (int64_t)((const char*)W3 - (const char*)W1);
    const int64_t ad = diff < 0 ? -diff : diff;
    if (ad == 0 || ad % 16 != 0 || ad >= (int64_t(1) << 40)) return 0;
    const uint64_t bk = 128 / es;
    const uint64_t dims[4] = {(uint64_t)d, (uint64_t)F, 2, (uint64_t)E};
    const uint64_t strides[3] = {(uint64_t)d * es, (uint64_t)ad, (uint64_t)estride * es};
    const uint32_t box[4] = {(uint32_t)bk, 128, 2, 1};
    if (!make_map_nd(m, diff > 0 ? W1 : W3, dt, 4, dims, strides, box)) return -1;
    return diff > 0 ? 1 : 2;
}

static int check_common(const void* A, const void* B, const int32_t* offsets, int64_t E,
                        int64_t R, int64_t d, int64_t F, int dtype) {
    if (E < 1 || E > MOE_MAX_EXPERTS || R < 0 || d <= 0 || F <= 0) return MOE_ERR_INVALID;
    if (dtype != MOE_BF16 && dtype != MOE_F32) return MOE_ERR_UNSUPPORTED;
    if (d % 128 != 0 || F % 128 != 0) return MOE_ERR_UNSUPPORTED;
    if (R > INT32_MAX - 2 * BM || d > (1 << 24) || F > (1 << 24)) return MOE_ERR_UNSUPPORTED;
    if (!offsets || !A || !B || !aligned16(A) || !aligned16(B)) return MOE_ERR_INVALID;
    return MOE_OK;
}

}  // namespace gg
}  // namespace moe

using namespace moe;

extern "C" int moe_grouped_gate_up_save(const void* Xe, const void* W1, const void* W3,
                                        int64_t w13_expert_stride, const int32_t* offsets,
                                        int64_t E, int64_t R, int64_t d, int64_t F, int dtype,
                                        void* H, void* A_out, void* B_out, void* stream) {
    if ((A_out == nullptr) != (B_out == nullptr)) return MOE_ERR_INVALID;
    if (A_out && (!aligned16(A_out) || !aligned16(B_out))) return MOE_ERR_INVALID;
    int rc = gg::check_common(Xe, W1, offsets, E, R, d, F, dtype);
    if (rc != MOE_OK) return rc;
    if (!W3 || !H || !aligned16(W3) || !aligned16(H)) return MOE_ERR_INVALID;
    if (w13_expert_stride < F * d && E > 1) return MOE_ERR_INVALID;
    if (w13_expert_stride % 8 != 0) return MOE_ERR_INVALID;
    if (R == 0) return MOE_OK;
    const int es = dtype == MOE_F32 ? 4 : 2;
    const CUtensorMapDataType dt =
        dtype == MOE_F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    CUtensorMap a, b0, b1;
    cudaStream_t st = as_stream(stream);
    if (gg::use_swap(R, E) && gg::gate_up_map_fits(W1, W3, w13_expert_stride, E, d, es)) {
        gg::sw::TokenMaps xm;
        int wpe = 0, second_is_gate = 0;
        if (!gg::make_gate_up_map(&b0, W1, W3, dt, es, w13_expert_stride, E, d, F, &wpe,
                                  &second_is_gate) ||
            !gg::make_token_maps(&xm, Xe, dt, es, d, R))
            return MOE_ERR_CUDA;
        if (dtype == MOE_BF16)
            return gg::launch_swap<__nv_bfloat16, true>(b0, xm, offsets, E, R, d, F, wpe,
                                                         second_is_gate, H, F, st, A_out, B_out);
        return gg::launch_swap<float, true>(b0, xm, offsets, E, R, d, F, wpe, second_is_gate, H, F,
                                            st, A_out, B_out);
    }
    if (!gg::make_map_2d(&a, Xe, dt, es, d, R, gg::BM)) return MOE_ERR_CUDA;
    const int b_mode = gg::make_w13_map(&b0, W1, W3, dt, es, w13_expert_stride, E, d, F);
    if (b_mode < 0) return MOE_ERR_CUDA;
    if (b_mode == 0 && (!gg::make_map_3d(&b0, W1, dt, es, d, F, E, w13_expert_stride, 128) ||
                        !gg::make_map_3d(&b1, W3, dt, es, d, F, E, w13_expert_stride, 128)))
        return MOE_ERR_CUDA;
    if (b_mode != 0) b1 = b0;
    if (dtype == MOE_BF16)
        return gg::launch<__nv_bfloat16, true, 256>(a, b0, b1, offsets, E, R, d, F, H, F, st,
                                                     A_out, B_out, nullptr, 0, b_mode);
    return gg::launch<float, true, 256>(a, b0, b1, offsets, E, R, d, F, H, F, st, A_out, B_out,
                                        nullptr, 0, b_mode);
}

extern "C" int moe_grouped_gate_up(const void* Xe, const void* W1, const void* W3,
                                   int64_t w13_expert_stride, const int32_t* offsets, int64_t E,
                                   int64_t R, int64_t d, int64_t F, int dtype, void* H,
                                   void* stream) {
    return moe_grouped_gate_up_save(Xe, W1, W3, w13_expert_stride, offsets, E, R, d, F, dtype, H,
                                    nullptr, nullptr, stream);
}

extern "C" int moe_grouped_gate_up_gather(const void* x, const int32_t* row_token, int64_t T,
                                          const void* W1, const void* W3,
                                          int64_t w13_expert_stride, const int32_t* offsets,
                                          int64_t E, int64_t R, int64_t d, int64_t F, int dtype,
                                          void* H, void* stream) {
    int rc = gg::check_common(x, W1, offsets, E, R, d, F, dtype);
    if (rc != MOE_OK) return rc;
    if (T < 0 || T > INT32_MAX || !row_token) return MOE_ERR_INVALID;
    if (!W3 || !H || !aligned16(W3) || !aligned16(H)) return MOE_ERR_INVALID;
    if (w13_expert_stride < F * d && E > 1) return MOE_ERR_INVALID;
    if (w13_expert_stride % 8 != 0) return MOE_ERR_INVALID;
    if (R == 0) return MOE_OK;
    if (T == 0) return MOE_ERR_INVALID;  // R rows but no token to gather
    const int es = dtype == MOE_F32 ? 4 : 2;
    const CUtensorMapDataType dt =
        dtype == MOE_F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    CUtensorMap a, b0, b1;
    if (!gg::make_map_2d(&a, x, dt, es, d, T, 1) ||  // one row high: gather4 boxes
        !gg::make_map_3d(&b0, W1, dt, es, d, F, E, w13_expert_stride, 128) ||
        !gg::make_map_3d(&b1, W3, dt, es, d, F, E, w13_expert_stride, 128))
        return MOE_ERR_CUDA;
    cudaStream_t st = as_stream(stream);
    if (dtype == MOE_BF16)
        return gg::launch<__nv_bfloat16, true, 256, true>(a, b0, b1, offsets, E, R, d, F, H, F, st,
                                                           nullptr, nullptr, row_token, T);
    return gg::launch<float, true, 256, true>(a, b0, b1, offsets, E, R, d, F, H, F, st, nullptr,
                                              nullptr, row_token, T);
}

static int grouped_down(const void* H, const void* W2, int64_t w2_expert_stride,
                        const int32_t* offsets, const float* row_gate, int64_t E, int64_t R,
                        int64_t d, int64_t F, int dtype, void* Ye, void* stream) {
    int rc = gg::check_common(H, W2, offsets, E, R, d, F, dtype);
    if (rc != MOE_OK) return rc;
    if (!Ye || !aligned16(Ye)) return MOE_ERR_INVALID;
    if (w2_expert_stride < F * d && E > 1) return MOE_ERR_INVALID;
    if (w2_expert_stride % 8 != 0) return MOE_ERR_INVALID;
    if (R == 0) return MOE_OK;
    const int es = dtype == MOE_F32 ? 4 : 2;
    const CUtensorMapDataType dt =
        dtype == MOE_F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const int mma_n = (d % 256 == 0) ? 256 : 128;
    CUtensorMap a, b0;
    if (mma_n == 256 && gg::use_swap(R, E) && gg::down_map_fits(w2_expert_stride, E, F)) {
        gg::sw::TokenMaps xm;
        int wpe = 0;
        if (!gg::make_down_map(&b0, W2, dt, es, w2_expert_stride, E, d, F, &wpe) ||
            !gg::make_token_maps(&xm, H, dt, es, F, R))
            return MOE_ERR_CUDA;
        cudaStream_t st = as_stream(stream);
        if (dtype == MOE_BF16)
            return gg::launch_swap<__nv_bfloat16, false>(b0, xm, offsets, E, R, F, d, wpe, 0, Ye, d,
                                                          st, nullptr, nullptr, row_gate);
        return gg::launch_swap<float, false>(b0, xm, offsets, E, R, F, d, wpe, 0, Ye, d, st,
                                             nullptr, nullptr, row_gate);
    }
    const bool pair = mma_n == 256 && gg::use_pair(R, E);
    if (!gg::make_map_2d(&a, H, dt, es, F, R, gg::BM) ||
        !gg::make_map_3d(&b0, W2, dt, es, F, d, E, w2_expert_stride, pair ? 128 : mma_n))
        return MOE_ERR_CUDA;
    cudaStream_t st = as_stream(stream);
    if (pair) {
        if (dtype == MOE_BF16)
            return gg::launch_pair<__nv_bfloat16, false>(a, b0, b0, offsets, E, R, F, d, Ye, d, st,
                                                          nullptr, nullptr, row_gate);
        return gg::launch_pair<float, false>(a, b0, b0, offsets, E, R, F, d, Ye, d, st, nullptr,
                                             nullptr, row_gate);
    }
    if (dtype == MOE_BF16) {
        if (mma_n == 256)
            return gg::launch<__nv_bfloat16, false, 256>(a, b0, b0, offsets, E, R, F, d, Ye, d, st,
                                                          nullptr, nullptr, nullptr, 0, 0, row_gate);
        return gg::launch<__nv_bfloat16, false, 128>(a, b0, b0, offsets, E, R, F, d, Ye, d, st,
                                                      nullptr, nullptr, nullptr, 0, 0, row_gate);
    }
    if (mma_n == 256)
        return gg::launch<float, false, 256>(a, b0, b0, offsets, E, R, F, d, Ye, d, st, nullptr,
                                             nullptr, nullptr, 0, 0, row_gate);
    return gg::launch<float, false, 128>(a, b0, b0, offsets, E, R, F, d, Ye, d, st, nullptr,
                                         nullptr, nullptr, 0, 0, row_gate);
}

extern "C" int moe_grouped_down(const void* H, const void* W2, int64_t w2_expert_stride,
                                const int32_t* offsets, int64_t E, int64_t R, int64_t d,
                                int64_t F, int dtype, void* Ye, void* stream) {
    return grouped_down(H, W2, w2_expert_stride, offsets, nullptr, E, R, d, F, dtype, Ye, stream);
}

extern "C" int moe_grouped_down_gated(const void* H, const void* W2, int64_t w2_expert_stride,
                                      const int32_t* offsets, const float* row_gate, int64_t E,
                                      int64_t R, int64_t d, int64_t F, int dtype, void* Ye,
                                      void* stream) {
    if (R > 0 && !row_gate) return MOE_ERR_INVALID;
    return grouped_down(H, W2, w2_expert_stride, offsets, row_gate, E, R, d, F, dtype, Ye, stream);
}

extern "C" int moe_debug_set_gemm_form(int form) {
    if (form < 0 || form > 2) return MOE_ERR_INVALID;
    gg::gemm_form() = form;
    return MOE_OK;
}

extern "C" int moe_grouped_swiglu(const void* Xe, const void* W1, const void* W3, const void* W2,
                                  int64_t w13_expert_stride, int64_t w2_expert_stride,
                                  const int32_t* offsets, int64_t E, int64_t R, int64_t d,
                                  int64_t F, int dtype, void* H, void* Ye, void* stream) {
    int rc = moe_grouped_gate_up(Xe, W1, W3, w13_expert_stride, offsets, E, R, d, F, dtype, H,
                                 stream);
    if (rc != MOE_OK) return rc;
    return moe_grouped_down(H, W2, w2_expert_stride, offsets, E, R, d, F, dtype, Ye, stream);
}
