// Backward of the grouped SwiGLU expert FFN on tcgen05 (sm_100a).
//
// For each expert e and its rows r in [offsets[e], offsets[e+1]), with the
// forward's pre-activations A = Xe W1_eᵀ, B = Xe W3_eᵀ, H = silu(A) * B and
// the upstream rows dYe (= gate * dOut[token], formed by the scaled dispatch):
//   dH  = dYe W2_e                               K = d
//   dA  = dH * B * silu'(A),  dB = dH * silu(A)  (pairwise SwiGLU backward,
//         fused into the dH epilogue; "OLMo-core 3 发布：主攻混合专家训练与导出校验",
//         主要功能: optional pairwise SwiGLU backward)
//   dXe = dA W1_e + dB W3_e                      K = 2F
//   dW1_e = dAᵀ Xe,  dW3_e = dBᵀ Xe,  dW2_e = dYeᵀ H   K = rows of e
// silu'(a) = s (1 + a (1 - s)), s = sigmoid(a). Weight gradients are written
// in bf16 from fp32 accumulators (the same release notes: bf16 weight
// gradients). The router and gate gradients are not part of this pass.
//
// One kernel template, three modes, the same pipeline as the forward grouped
// GEMM (TMA producer warp, single-thread tcgen05.mma issue, 4 epilogue warps,
// 4-stage shared-memory ring, double-buffered 128x256 fp32 TMEM accumulator,
// 8 epilogue warps: each TMEM lane quarter is drained by two warps, one per
// half of the columns):
//   DH  A = dYe rows (K-major), B = W2_e read as [F x d] (MN-major, F
//       contiguous); epilogue loads A,B of the same rows/columns and writes dA, dB.
//   DX  A = dA then dB rows (K-major), B = W1_e then W3_e read as [d x F]
//       (MN-major, d contiguous); epilogue writes dXe.
//   DW  per expert a 128 x 256 tile of the [M x N] gradient; A and B are the
//       expert's rows of two [R x M] / [R x N] matrices, both MN-major, with K
//       running over the rows. The last K slab of an expert can reach into the
//       next expert's rows: only its 16-row MMA steps that hold valid rows run,
//       and the few foreign rows inside the last of them are zeroed in shared
//       memory before the MMA reads them. An expert with no rows writes zeros.
#include "tc_sm100.cuh"

namespace moe {
namespace bwd {

using namespace tc;

constexpr int BM = 128;
constexpr int MMA_N = 256;
constexpr int BK = 64;  // bf16 elements per 128-byte slab
constexpr int EPI_WARPS = 8;  // two per TMEM lane quarter, one per column half
constexpr int THREADS = 64 + 32 * EPI_WARPS;
constexpr int A_BYTES = BM * 128;
constexpr int B_BYTES = MMA_N * 128;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int BOX_BYTES = 64 * 128;  // one MN-major box: 64 K rows x 64 elements
constexpr int TMEM_ALLOC = 512;
constexpr int STG_BYTES = 32 * 128;  // dW store staging: 32 rows x 64 bf16, one per buffer

// DXR and DWF serve the router GEMM backward (one row group, or token chunks
// as groups): DXR is DH's operand layout with an epilogue that adds the
// product into the existing out0 rows; DWF is DW with fp32 output tiles (the
// partials of a split-K sum).
enum Mode { DH = 0, DX = 1, DW = 2, DXR = 3, DWF = 4, DWS = 5 };
template <int MODE>
constexpr bool is_dw() { return MODE == DW || MODE == DWF || MODE == DWS; }

// DW tiles have a short K (an expert's rows) and a large output. With 128
// or more rows per expert, the load ring keeps 4 stages like the other modes
// (a tile's K loop is a few slabs, so the ring's depth is what keeps bytes
// in flight) and each epilogue warp has one staging buffer for its TMA
// tensor stores; with fewer rows (DWS) a tile is one or two slabs and the
// stores bound it, so 3 stages and 2 staging buffers per warp. The expert
// offsets are read from global memory instead of a shared table. (One 8 KB
// store per warp and tile instead of two 4 KB ones needs the room of a
// load stage and measured slower on B200: the 4th stage is what lets the
// next tile's loads run ahead.)
template <int MODE>
struct ModeCfg {
    static constexpr bool A_MN = is_dw<MODE>();
    static constexpr uint32_t IDESC = make_idesc_major(1u, BM, MMA_N, A_MN, true);
    static constexpr int STAGES = MODE == DWS ? 3 : 4;
    static constexpr int STG_BUFS = MODE == DWS ? 2 : (is_dw<MODE>() ? 1 : 0);  // per epilogue warp
    static constexpr int STAGING = EPI_WARPS * STG_BUFS * STG_BYTES;
    static constexpr bool TABLES = !is_dw<MODE>();  // shared offset and tile tables
    static constexpr int NUM_BARS = 2 * STAGES + 5;
    static constexpr int META_BYTES =
        NUM_BARS * 8 + 16 + (TABLES ? 2 * 4 * (MOE_MAX_EXPERTS + 1) : 0);
    static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + STAGING + META_BYTES;
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
};

struct Tile {
    int e, row0, row_end, m0, n0, kb0, nkb;
};

__device__ __forceinline__ float sigmoidf_(float a) { return 1.0f / (1.0f + __expf(-a)); }

template <int MODE>
__device__ __forceinline__ Tile decode(int t, int E, int NB, int MB, int K, const int* s_toff,
                                       const int* s_off) {
    Tile tl;
    if (is_dw<MODE>()) {
        const int tpe = MB * NB;
        const int e = t / tpe;
        const int l = t - e * tpe;
        const int nb = l / MB, mb = l - nb * MB;
        tl.e = e;
        tl.row0 = s_off[e];
        tl.row_end = s_off[e + 1];
        tl.m0 = mb * BM;
        tl.n0 = nb * MMA_N;
        tl.kb0 = 0;
        tl.nkb = (tl.row_end - tl.row0 + BK - 1) / BK;
    } else {
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
        tl.e = lo;
        tl.row0 = s_off[lo] + m * BM;
        tl.row_end = s_off[lo + 1];
        tl.m0 = 0;
        tl.n0 = nb * MMA_N;
        tl.kb0 = 0;
        tl.nkb = K / BK;
    }
    return tl;
}

__device__ __forceinline__ void store32_bf16(__nv_bfloat16* dst, const float* v) {
    uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
    for (int i = 0; i < 4; ++i) d[i] = pack8(v + 8 * i);
}

__device__ __forceinline__ void load32_bf16(const __nv_bfloat16* src, float* v) {
    const uint4* s = reinterpret_cast<const uint4*>(src);
#pragma unroll
    for (int i = 0; i < 4; ++i) unpack8(__ldg(s + i), v + 8 * i);
}

// tmA0/tmA1/tmB0/tmB1: see the mode table at the top of the file.
//   K      DH: d; DX: 2F (KF = K/2 slabs per operand pair); DW: unused
//   Mdim   DW: rows of each expert's gradient (F or d)
//   Ndim   DH: F; DX: d; DW: columns of each expert's gradient
//   tmOut  DW: the gradient viewed as [E*Mdim, Ndim] bf16, box 64 x 32 (TMA store)
template <int MODE>
__global__ void __launch_bounds__(THREADS, 1)
    bwd_gemm_kernel(const __grid_constant__ CUtensorMap tmA0,
                    const __grid_constant__ CUtensorMap tmA1,
                    const __grid_constant__ CUtensorMap tmB0,
                    const __grid_constant__ CUtensorMap tmB1,
                    const __grid_constant__ CUtensorMap tmOut,
                    const int32_t* __restrict__ offsets, int E, int R, int K, int Mdim, int Ndim,
                    __nv_bfloat16* __restrict__ out0, __nv_bfloat16* __restrict__ out1,
                    int64_t ldo, const __nv_bfloat16* __restrict__ saveA,
                    const __nv_bfloat16* __restrict__ saveB, int* status) {
    using C = ModeCfg<MODE>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    constexpr int STAGES = C::STAGES;
    constexpr int NUM_BARS = C::NUM_BARS;
    uint8_t* staging = smem + STAGES * STAGE_BYTES;
    uint8_t* meta = staging + C::STAGING;
    uint64_t* bars = reinterpret_cast<uint64_t*>(meta);
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(meta + NUM_BARS * 8);
    volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
    int* s_bad = reinterpret_cast<int*>(s_tmem + 2);
    // DW: the offsets straight from global memory; the others: shared copies
    // and the tile table
    int* s_tab = reinterpret_cast<int*>(meta + NUM_BARS * 8 + 16);
    const int* s_off = C::TABLES ? s_tab : offsets;
    int* s_toff = C::TABLES ? s_tab + (MOE_MAX_EXPERTS + 1) : nullptr;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint64_t wl = wait_limit();  // the pipeline waits' time limit, read once

    // --- routing offsets -> tile table (validated) -----------------------
    if (C::TABLES)
        for (int e = tid; e <= E; e += THREADS) s_tab[e] = offsets[e];
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
            if (C::TABLES && e < E) s_toff[e] = carry + ex;
            carry += tot;
        }
        bad = __any_sync(0xffffffffu, bad) || s_off[0] != 0 || s_off[E] != R;
        if (lane == 0) {
            if (C::TABLES) s_toff[E] = carry;
            *s_bad = bad ? 1 : 0;
        }
    }
    __syncthreads();
    if (*s_bad) {
        if (tid == 0 && blockIdx.x == 0) set_status(status, MOE_DEVERR_BAD_OFFSETS);
        return;
    }
    const int NB = Ndim / MMA_N;
    const int MB = is_dw<MODE>() ? Mdim / BM : 1;
    const int total = is_dw<MODE>() ? E * MB * NB : s_toff[E] * NB;
    if ((int)blockIdx.x >= total) return;
    const int KF = K / 2 / BK;  // DX: slabs per operand pair

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
        prefetch_map(&tmA0);
        prefetch_map(&tmB0);
        if (MODE == DX) {
            prefetch_map(&tmA1);
            prefetch_map(&tmB1);
        }
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(s_tmem), TMEM_ALLOC);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *s_tmem;

    if (warp == 0 && lane == 0) {
        // ------------------------------------------------ TMA producer
        int stage = 0;
        uint32_t phase = 0, issued_mask = 0, issued_parity = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
            const Tile tl = decode<MODE>(t, E, NB, MB, K, s_toff, s_off);
            for (int kb = 0; kb < tl.nkb; ++kb) {
                if (!mbar_wait(smem_u32(empty + stage), phase ^ 1u, s_abort, status, wl)) {
                    ok = false;
                    break;
                }
                const uint32_t fb = smem_u32(full + stage);
                const uint32_t sa = smem_u32(smem + stage * STAGE_BYTES);
                const uint32_t sb = sa + A_BYTES;
                mbar_expect_tx(fb, STAGE_BYTES);
                // one copy per operand: the MN-major operands' 64-column
                // boxes come as the chunks of one box of a map whose third
                // dimension steps 64 columns (few large copies stream faster
                // than many small ones on B200)
                if (MODE == DH || MODE == DXR) {
                    tma_load_2d(sa, &tmA0, fb, kb * BK, tl.row0);
                    tma_load_4d(sb, &tmB0, fb, 0, kb * BK, tl.n0 / 64, tl.e);
                } else if (MODE == DX) {
                    const bool second = kb >= KF;
                    const int kf = second ? kb - KF : kb;
                    tma_load_2d(sa, second ? &tmA1 : &tmA0, fb, kf * BK, tl.row0);
                    tma_load_4d(sb, second ? &tmB1 : &tmB0, fb, 0, kf * BK, tl.n0 / 64, tl.e);
                } else {
                    const int r = tl.row0 + kb * BK;
                    tma_load_3d(sa, &tmA0, fb, 0, r, tl.m0 / 64);
                    tma_load_3d(sb, &tmB0, fb, 0, r, tl.n0 / 64);
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
            for (int s = 0; s < STAGES; ++s)
                if ((issued_mask >> s) & 1u) {
                    volatile int no_abort = 0;
                    mbar_wait(smem_u32(full + s), (issued_parity >> s) & 1u, &no_abort, nullptr,
                              DRAIN_LIMIT_NS);
                }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer (whole warp;
        // lane 0 issues, all lanes zero out-of-segment rows in DW mode)
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        int i = 0;
        for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++i) {
            const Tile tl = decode<MODE>(t, E, NB, MB, K, s_toff, s_off);
            const int buf = i & 1;
            const uint32_t tp = (uint32_t)(i >> 1) & 1u;
            if (!mbar_wait(smem_u32(tempty + buf), tp ^ 1u, s_abort, status, wl)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t dt = tmem_base + (uint32_t)(buf * MMA_N);
            for (int kb = 0; kb < tl.nkb; ++kb) {
                if (!mbar_wait(smem_u32(full + stage), phase, s_abort, status, wl)) {
                    ok = false;
                    break;
                }
                uint8_t* sa_p = smem + stage * STAGE_BYTES;
                const uint32_t sa = smem_u32(sa_p);
                const uint32_t sb = sa + A_BYTES;
                int nks = 4;  // 16-row K steps of this slab the MMAs consume
                if (is_dw<MODE>()) {
                    const int valid = tl.row_end - (tl.row0 + kb * BK);
                    if (valid < BK) {
                        // The slab ends inside the expert's last rows: only the K
                        // steps holding valid rows run, and the rows between the
                        // last valid row and the end of its 16-row step (another
                        // expert's rows, or past R) are zeroed in all 6 boxes first.
                        nks = (valid + 15) >> 4;
                        const int nz = nks * 16 - valid;
                        if (nz > 0) {
#pragma unroll 1
                            for (int box = 0; box < 6; ++box)
                                for (int c = lane; c < nz * 8; c += 32) {
                                    uint8_t* p = sa_p + box * BOX_BYTES + (valid + (c >> 3)) * 128 +
                                                 ((c & 7) << 4);
                                    *reinterpret_cast<uint4*>(p) = make_uint4(0, 0, 0, 0);
                                }
                            fence_proxy_async_smem();
                        }
                        __syncwarp();
                    }
                }
                if (lane == 0) {
                    tc_fence_after();
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks) {
                        if (ks >= nks) break;
                        const uint64_t ad = C::A_MN ? sw128_mn_desc(sa + ks * 2048, BOX_BYTES)
                                                    : sw128_desc(sa) + 2 * ks;
                        const uint64_t bd = sw128_mn_desc(sb + ks * 2048, BOX_BYTES);
                        tc_mma<false>(dt, ad, bd, C::IDESC, (kb | ks) != 0);
                    }
                    tc_commit(smem_u32(empty + stage));
                }
                __syncwarp();
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (ok && lane == 0) tc_commit(smem_u32(tfull + buf));
            __syncwarp();
        }
        if (!ok && lane == 0) {
            tc_commit(smem_u32(drain));
            volatile int no_abort = 0;
            mbar_wait(smem_u32(drain), 0, &no_abort, nullptr, DRAIN_LIMIT_NS);
        }
        __syncwarp();
    } else if (warp >= 2) {
        // ------------------------------------------------ epilogue
        const int q = warp & 3;                       // TMEM lane quarter
        const int col0 = ((warp - 2) >> 2) * (MMA_N / 2);  // this warp's column half
        const int r_in_tile = q * 32 + lane;
        int stg_count = 0;
        int i = 0;
        for (int t = blockIdx.x; t < total; t += gridDim.x, ++i) {
            const Tile tl = decode<MODE>(t, E, NB, MB, K, s_toff, s_off);
            const int buf = i & 1;
            const uint32_t tp = (uint32_t)(i >> 1) & 1u;
            if (!mbar_wait(smem_u32(tfull + buf), tp, s_abort, status, wl)) break;
            tc_fence_after();
            const uint32_t ta = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * MMA_N);
            if constexpr (MODE == DWF) {
                // 32-column groups: TMEM -> fp32 -> 128-byte-swizzled staging
                // (chunk c of row r at c ^ (r % 8)) -> TMA store of the warp's
                // 32 x 32 fp32 box; one staging buffer per warp
                const bool empty_k = tl.nkb == 0;
                const int ybase = tl.e * Mdim + tl.m0 + q * 32;
                uint8_t* stg = staging + (warp - 2) * C::STG_BUFS * STG_BYTES;
#pragma unroll 1
                for (int cc = col0 / 32; cc < (col0 + MMA_N / 2) / 32; ++cc) {
                    uint8_t* sbuf = stg + (stg_count % C::STG_BUFS) * STG_BYTES;
                    ++stg_count;
                    if (lane == 0) bulk_wait_read<C::STG_BUFS - 1>();  // its previous store has read it
                    __syncwarp();
                    uint32_t a[32];
                    if (!empty_k) {
                        tmem_ld32(ta + cc * 32, a);
                        tmem_wait_ld();
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; ++j) a[j] = 0u;
                    }
#pragma unroll
                    for (int chunk = 0; chunk < 8; ++chunk)
                        *reinterpret_cast<uint4*>(sbuf + lane * 128 + ((chunk ^ (lane & 7)) << 4)) =
                            make_uint4(a[4 * chunk], a[4 * chunk + 1], a[4 * chunk + 2],
                                       a[4 * chunk + 3]);
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_2d(&tmOut, smem_u32(sbuf), tl.n0 + cc * 32, ybase);
                        bulk_commit();
                    }
                }
            } else if constexpr (MODE == DW || MODE == DWS) {
                // 64-column groups: TMEM -> bf16 -> 128-byte-swizzled staging
                // (chunk c of row r at c ^ (r % 8), conflict-free) -> TMA store
                // of the warp's 32 x 64 box; one staging buffer per warp
                const bool empty_k = tl.nkb == 0;
                const int ybase = tl.e * Mdim + tl.m0 + q * 32;
                uint8_t* stg = staging + (warp - 2) * C::STG_BUFS * STG_BYTES;
#pragma unroll 1
                for (int cc = col0 / 64; cc < (col0 + MMA_N / 2) / 64; ++cc) {
                    uint8_t* sbuf = stg + (stg_count % C::STG_BUFS) * STG_BYTES;
                    ++stg_count;
                    if (lane == 0) bulk_wait_read<C::STG_BUFS - 1>();  // its previous store has read it
                    __syncwarp();
                    uint32_t a[2][32];
                    if (!empty_k) {
                        tmem_ld32(ta + cc * 64, a[0]);
                        tmem_ld32(ta + cc * 64 + 32, a[1]);
                        tmem_wait_ld();
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; ++j) a[0][j] = a[1][j] = 0u;
                    }
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const int chunk = h * 4 + j;
                            *reinterpret_cast<uint4*>(sbuf + lane * 128 + ((chunk ^ (lane & 7)) << 4)) =
                                pack8(reinterpret_cast<const float*>(a[h]) + 8 * j);
                        }
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_2d(&tmOut, smem_u32(sbuf), tl.n0 + cc * 64, ybase);
                        bulk_commit();
                    }
                }
            } else {
                const int grow = tl.row0 + r_in_tile;
                const bool valid = grow < tl.row_end;
                const size_t rowoff = (size_t)(valid ? grow : 0) * ldo + tl.n0;
#pragma unroll 1
                for (int c = col0 / 32; c < (col0 + MMA_N / 2) / 32; ++c) {
                    uint32_t a[32];
                    tmem_ld32(ta + c * 32, a);
                    tmem_wait_ld();
                    if (!valid) continue;
                    float v[32];
#pragma unroll
                    for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(a[j]);
                    if (MODE == DXR) {
                        float old[32];
                        load32_bf16(out0 + rowoff + c * 32, old);
#pragma unroll
                        for (int j = 0; j < 32; ++j) v[j] += old[j];
                        store32_bf16(out0 + rowoff + c * 32, v);
                    } else if (MODE == DH) {
                        float ga[32], ub[32], da[32], db[32];
                        load32_bf16(saveA + rowoff + c * 32, ga);
                        load32_bf16(saveB + rowoff + c * 32, ub);
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const float s = sigmoidf_(ga[j]);
                            const float silu = ga[j] * s;
                            const float dsilu = s * (1.0f + ga[j] * (1.0f - s));
                            da[j] = v[j] * ub[j] * dsilu;
                            db[j] = v[j] * silu;
                        }
                        store32_bf16(out0 + rowoff + c * 32, da);
                        store32_bf16(out1 + rowoff + c * 32, db);
                    } else {
                        store32_bf16(out0 + rowoff + c * 32, v);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(tempty + buf));
        }
        if (is_dw<MODE>() && lane == 0) bulk_wait<0>();  // stores done before the CTA leaves
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) {
        __syncwarp();
        tmem_dealloc(tmem_base, TMEM_ALLOC);
    }
}

template <int MODE>
static int launch(const CUtensorMap& a0, const CUtensorMap& a1, const CUtensorMap& b0,
                  const CUtensorMap& b1, const CUtensorMap& om, const int32_t* offsets, int64_t E,
                  int64_t R, int64_t K, int64_t Mdim, int64_t Ndim, void* out0, void* out1,
                  int64_t ldo, const void* saveA, const void* saveB, cudaStream_t st) {
    auto kern = bwd_gemm_kernel<MODE>;
    constexpr int SMEM_BYTES = ModeCfg<MODE>::SMEM_BYTES;
    if (check_only()) return MOE_OK;
    static bool attr_done[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_done[dev]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES) !=
            cudaSuccess)
            return MOE_ERR_CUDA;
        attr_done[dev] = true;
    }
    const int64_t NB = Ndim / MMA_N;
    const int64_t max_tiles = is_dw<MODE>() ? E * (Mdim / BM) * NB : (R / BM + E) * NB;
    const int64_t sms = num_sms();
    const int grid = (int)(max_tiles < sms ? max_tiles : sms);
    if (grid <= 0) return MOE_OK;
    kern<<<grid, THREADS, SMEM_BYTES, st>>>(
        a0, a1, b0, b1, om, offsets, (int)E, (int)R, (int)K, (int)Mdim, (int)Ndim,
        static_cast<__nv_bfloat16*>(out0), static_cast<__nv_bfloat16*>(out1), ldo,
        static_cast<const __nv_bfloat16*>(saveA), static_cast<const __nv_bfloat16*>(saveB),
        status_ptr());
    return launch_status();
}

constexpr CUtensorMapDataType BF16 = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;

// MN-major operand map over bf16 [rows, cols] (E == 0) or E such matrices
// `estride` elements apart: dims (64 columns, rows, cols / 64 chunks[, E]),
// so one box of `chunks` chunks x 64 rows lands as `chunks` consecutive
// 64-row x 128-byte tiles, the layout the MN-major MMA descriptors read.
inline bool make_mn_map(CUtensorMap* m, const void* base, int64_t cols, int64_t rows, int64_t E,
                        int64_t estride, uint32_t chunks) {
    const uint64_t dims[4] = {64, (uint64_t)rows, (uint64_t)cols / 64, (uint64_t)(E > 0 ? E : 1)};
    const uint64_t strides[3] = {(uint64_t)cols * 2, 128, (uint64_t)(E > 0 ? estride : 0) * 2};
    const uint32_t box[4] = {64, 64, chunks, 1};
    return tc::make_map_nd(m, base, BF16, E > 0 ? 4 : 3, dims, strides, box);
}

}  // namespace bwd
}  // namespace moe

namespace moe {

// Router GEMM backward on the tensor cores, for router_bwd.cu. dl: dlogits in
// bf16, [T, Ep] with Ep = E rounded up to 64 and zeros past E. dx (if not
// null) += dl Wr: DXR over one row group (off_one = {0, T}), K = Ep, with Wr
// [E, d] read MN-major (rows past E read as zeros). partial (if not null):
// for token chunk g (off_chunks, G chunks), rows 0..Mp-1 of dlᵀ x over the
// chunk's tokens, fp32 [G*Mp, d] (DWF, M = Mp = Ep rounded up to 128, columns
// of dl past Ep read as zeros). d % 256 == 0.
int router_linear_bwd_tc(const void* dl, int64_t Ep, const void* x, const void* Wr, int64_t T,
                         int64_t d, int64_t E, const int32_t* off_one, const int32_t* off_chunks,
                         int64_t G, int64_t Mp, void* dx, float* partial, cudaStream_t st) {
    using namespace tc;
    if (dx) {
        CUtensorMap ma, mb;
        if (!make_map_2d(&ma, dl, bwd::BF16, 2, Ep, T, bwd::BM) ||
            !bwd::make_mn_map(&mb, Wr, d, E, 1, E * d, 4))
            return MOE_ERR_CUDA;
        const int rc = bwd::launch<bwd::DXR>(ma, ma, mb, mb, ma, off_one, 1, T, Ep, 0, d, dx,
                                             nullptr, d, nullptr, nullptr, st);
        if (rc != MOE_OK) return rc;
    }
    if (partial) {
        CUtensorMap ma, mb, mo;
        if (!bwd::make_mn_map(&ma, dl, Ep, T, 0, 0, 2) || !bwd::make_mn_map(&mb, x, d, T, 0, 0, 4) ||
            !make_map_2d(&mo, partial, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, d, G * Mp, 32))
            return MOE_ERR_CUDA;
        return bwd::launch<bwd::DWF>(ma, ma, mb, mb, mo, off_chunks, G, T, 0, Mp, d, nullptr,
                                     nullptr, d, nullptr, nullptr, st);
    }
    return MOE_OK;
}


// Weight gradients of the grouped SwiGLU FFN from bf16 rows: dW1_e = dAᵀ Xe,
// dW3_e = dBᵀ Xe, dW2_e = dYeᵀ H over each expert's rows (every expert's
// tiles run, so an expert with no rows gets zeros). Shared by the bf16 and
// the MXFP8 backward (there Xe and H are the dequantised forward operands).
int swiglu_wgrad(const void* Xe, const void* dA, const void* dB, const void* dYe, const void* H,
                 const int32_t* offsets, int64_t E, int64_t R, int64_t d, int64_t F, void* dW1,
                 void* dW3, void* dW2, cudaStream_t st) {
    using namespace tc;
    CUtensorMap gA, gB, gX, gY, gH;
    const int64_t Rm = R > 0 ? R : 1;  // a map needs a non-empty extent; no rows are read when R == 0
    // A operands (M side, 2 chunks = 128 columns) and B operands (N side, 4
    // chunks = 256 columns) of the weight-gradient tiles
    if (!bwd::make_mn_map(&gA, dA, F, Rm, 0, 0, 2) || !bwd::make_mn_map(&gB, dB, F, Rm, 0, 0, 2) ||
        !bwd::make_mn_map(&gY, dYe, d, Rm, 0, 0, 2) || !bwd::make_mn_map(&gX, Xe, d, Rm, 0, 0, 4) ||
        !bwd::make_mn_map(&gH, H, F, Rm, 0, 0, 4))
        return MOE_ERR_CUDA;
    CUtensorMap o1, o3, o2;  // the gradients as [E*M, N] for the TMA stores
    if (!make_map_2d(&o1, dW1, bwd::BF16, 2, d, E * F, 32) ||
        !make_map_2d(&o3, dW3, bwd::BF16, 2, d, E * F, 32) ||
        !make_map_2d(&o2, dW2, bwd::BF16, 2, F, E * d, 32))
        return MOE_ERR_CUDA;
    if (R < 128 * E) {  // experts average fewer than 128 rows: the store-bound form
        int rc = bwd::launch<bwd::DWS>(gA, gA, gX, gX, o1, offsets, E, R, 0, F, d, dW1, nullptr,
                                       d, nullptr, nullptr, st);
        if (rc != MOE_OK) return rc;
        rc = bwd::launch<bwd::DWS>(gB, gB, gX, gX, o3, offsets, E, R, 0, F, d, dW3, nullptr, d,
                                   nullptr, nullptr, st);
        if (rc != MOE_OK) return rc;
        return bwd::launch<bwd::DWS>(gY, gY, gH, gH, o2, offsets, E, R, 0, d, F, dW2, nullptr, F,
                                     nullptr, nullptr, st);
    }
    int rc = bwd::launch<bwd::DW>(gA, gA, gX, gX, o1, offsets, E, R, 0, F, d, dW1, nullptr, d,
                                  nullptr, nullptr, st);
    if (rc != MOE_OK) return rc;
    rc = bwd::launch<bwd::DW>(gB, gB, gX, gX, o3, offsets, E, R, 0, F, d, dW3, nullptr, d, nullptr,
                              nullptr, st);
    if (rc != MOE_OK) return rc;
    return bwd::launch<bwd::DW>(gY, gY, gH, gH, o2, offsets, E, R, 0, d, F, dW2, nullptr, F,
                                nullptr, nullptr, st);
}
}  // namespace moe

using namespace moe;
using namespace moe::tc;

extern "C" int moe_grouped_swiglu_bwd(const void* Xe, const void* A, const void* B, const void* H,
                                      const void* dYe, const void* W1, const void* W3,
                                      const void* W2, int64_t w13_expert_stride,
                                      int64_t w2_expert_stride, const int32_t* offsets, int64_t E,
                                      int64_t R, int64_t d, int64_t F, int dtype, void* dA,
                                      void* dB, void* dXe, void* dW1, void* dW3, void* dW2,
                                      void* stream) {
    if (E < 1 || E > MOE_MAX_EXPERTS || R < 0 || d <= 0 || F <= 0) return MOE_ERR_INVALID;
    if (dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
    if (d % 256 != 0 || F % 256 != 0) return MOE_ERR_UNSUPPORTED;
    if (R > INT32_MAX - 2 * bwd::BM || d > (1 << 24) || F > (1 << 24)) return MOE_ERR_UNSUPPORTED;
    const void* ptrs[] = {Xe, A, B, H, dYe, W1, W3, W2, dA, dB, dXe, dW1, dW3, dW2};
    for (const void* p : ptrs)
        if (!p || !aligned16(p)) return MOE_ERR_INVALID;
    if (!offsets) return MOE_ERR_INVALID;
    if ((w13_expert_stride < F * d || w2_expert_stride < F * d) && E > 1) return MOE_ERR_INVALID;
    if (w13_expert_stride % 8 != 0 || w2_expert_stride % 8 != 0) return MOE_ERR_INVALID;
    cudaStream_t st = as_stream(stream);
    int rc;
    if (R > 0) {
        // dH = dYe W2_e (+ pairwise SwiGLU backward) -> dA, dB
        CUtensorMap mA, mW2;
        if (!make_map_2d(&mA, dYe, bwd::BF16, 2, d, R, bwd::BM) ||
            !bwd::make_mn_map(&mW2, W2, F, d, E, w2_expert_stride, 4))
            return MOE_ERR_CUDA;
        rc = bwd::launch<bwd::DH>(mA, mA, mW2, mW2, mA, offsets, E, R, d, 0, F, dA, dB, F, A, B,
                                  st);
        if (rc != MOE_OK) return rc;
        // dXe = dA W1_e + dB W3_e
        CUtensorMap mdA, mdB, mW1, mW3;
        if (!make_map_2d(&mdA, dA, bwd::BF16, 2, F, R, bwd::BM) ||
            !make_map_2d(&mdB, dB, bwd::BF16, 2, F, R, bwd::BM) ||
            !bwd::make_mn_map(&mW1, W1, d, F, E, w13_expert_stride, 4) ||
            !bwd::make_mn_map(&mW3, W3, d, F, E, w13_expert_stride, 4))
            return MOE_ERR_CUDA;
        rc = bwd::launch<bwd::DX>(mdA, mdB, mW1, mW3, mdA, offsets, E, R, 2 * F, 0, d, dXe,
                                  nullptr, d, nullptr, nullptr, st);
        if (rc != MOE_OK) return rc;
    }
    // weight gradients (every expert's tile runs, so empty experts get zeros)
    return swiglu_wgrad(Xe, dA, dB, dYe, H, offsets, E, R, d, F, dW1, dW3, dW2, st);
}

extern "C" int moe_grouped_swiglu_wgrad(const void* Xe, const void* dA, const void* dB,
                                        const void* dYe, const void* H, const int32_t* offsets,
                                        int64_t E, int64_t R, int64_t d, int64_t F, int dtype,
                                        void* dW1, void* dW3, void* dW2, void* stream) {
    if (E < 1 || E > MOE_MAX_EXPERTS || R < 0 || d <= 0 || F <= 0) return MOE_ERR_INVALID;
    if (dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
    if (d % 256 != 0 || F % 256 != 0) return MOE_ERR_UNSUPPORTED;
    if (R > INT32_MAX - 2 * bwd::BM || d > (1 << 24) || F > (1 << 24)) return MOE_ERR_UNSUPPORTED;
    const void* ptrs[] = {Xe, dA, dB, dYe, H, dW1, dW3, dW2};
    for (const void* p : ptrs)
        if (!p || !aligned16(p)) return MOE_ERR_INVALID;
    if (!offsets) return MOE_ERR_INVALID;
    return swiglu_wgrad(Xe, dA, dB, dYe, H, offsets, E, R, d, F, dW1, dW3, dW2, as_stream(stream));
}
