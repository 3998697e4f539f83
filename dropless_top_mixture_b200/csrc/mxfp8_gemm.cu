// MXFP8 variant of the layer: dispatch that quantises each token row once,
// and the grouped SwiGLU FFN on block-scaled FP8 tensor cores (sm_100a).
//
// "olmoforge" README, capability table and "MXFP8 分块量化": 32-value blocks
// share one scale, E4M3 payload; the Olmo-core 3 news article (xxqk.cn),
// "三招拆分、三项优化、一个精度开关": MXFP8 as the low-precision switch, its
// gain coming from the FFN and the expert data movement. Operands here:
//   x  -> Xq [R,d] e4m3 + UE8M0 scales [R,d/32]   (moe_dispatch_mxfp8)
//   W1, W3 [E,F,d], W2 [E,d,F] quantised offline along their K dimension
//   H  -> Hq [R,F] e4m3 + scales [R,F/32], quantised from the fp32 SwiGLU
//         output in the gate/up epilogue
//   Ye = Hq W2q (block-scaled), fp32 accumulate, bf16 out; combine as in bf16.
//
// Kernel: tcgen05.mma kind::mxf8f6f4.block_scale, M = 128, N = 256, K = 32 per
// instruction, 128-byte K slabs staged by TMA with the same 128-byte swizzle
// as the bf16 kernels, one slab (4 MMAs) per stage, four stages. The wide N
// halves the A traffic per flop against N = 128 and lets four 48 KB stages
// be in flight: the operands of a 256-row expert come from DRAM (each weight
// tile serves two row tiles), so bytes in flight bound the rate. Per slab
// every row carries 4 UE8M0 scales (one 32-bit word); the producer warp
// gathers the 128 A words (cp.async, tracked by the stage's mbarrier) and
// fetches the B words pre-packed (mxfp8_pack_weight_scales) with one bulk
// copy, both in the 32-row x 16-byte layout that tcgen05.cp.32x128b.warpx4
// copies into TMEM (lane m%32 of every sub-partition, column m/32, byte = K
// block); the MMA selects the byte with the scale-factor id of each of its
// 4 MMAs. TMEM: one 256-column accumulator (two would leave no room for the
// scale factors), then the scale factors. Eight epilogue warps first load
// their 128 accumulator columns into registers and release the accumulator,
// so the next tile's MMAs overlap the quantisation and stores.
#include "mx_common.cuh"
#include "tc_sm100.cuh"

namespace moe {
namespace mxg {

using namespace tc;

constexpr int BM = 128;
constexpr int MMA_N = 256;
constexpr int BK = 128;  // e4m3 elements per 128-byte slab (one slab per stage)
constexpr int STAGES = 4;
constexpr int EPI_WARPS = 8;
constexpr int THREADS = 64 + 32 * EPI_WARPS;
constexpr int A_BYTES = BM * 128;
constexpr int B_BYTES = MMA_N * 128;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int SF_BLOCK = 512;  // scale words of 128 rows for one slab
// per stage: the A block, then the two B blocks (contiguous, so one bulk copy
// brings the packed weight scales of the stage)
constexpr int SF_STAGE_BYTES = 3 * SF_BLOCK;
constexpr int TMEM_ALLOC = 512;
constexpr int SFA_COL = MMA_N;        // 256..259
constexpr int SFB_COL = SFA_COL + 4;  // 260..267
constexpr int NUM_BARS = 2 * STAGES + 3;
constexpr int META_BYTES = NUM_BARS * 8 + 16 + 2 * 4 * (MOE_MAX_EXPERTS + 1);
constexpr int SMEM_BYTES = 1024 + STAGES * (STAGE_BYTES + SF_STAGE_BYTES) + META_BYTES;
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");

// Block-scaled instruction descriptor: E4M3 A and B (format 0), K-major,
// N >> 3 at bit 17, UE8M0 scales (bit 23), M >> 4 at bit 24, scale-factor
// ids of A (bits 29-30) and B (bits 4-5) select the byte of the scale word.
__host__ __device__ constexpr uint32_t mx_idesc(int sf_id) {
    return ((uint32_t)sf_id << 4) | ((uint32_t)(MMA_N >> 3) << 17) | (1u << 23) |
           ((uint32_t)(BM >> 4) << 24) | ((uint32_t)sf_id << 29);
}

__device__ __forceinline__ void mma_mx(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                       uint32_t accum) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
            d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accum), "r"(sfa), "r"(sfb)
        : "memory");
}

// 32 rows x 16 bytes, contiguous, no swizzle: 8-row core matrices 128 bytes apart.
__device__ __forceinline__ uint64_t sf_desc(uint32_t saddr) {
    return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)(128 >> 4) << 32) |
           ((uint64_t)1 << 46);
}

__device__ __forceinline__ void tmem_cp_sf(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
                 : "memory");
}

struct Tile {
    int e, row0, row_end, n0;
    int tile;  // global row-tile index: s_toff[e] + row tile within the expert
};

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
    tl.tile = s_toff[lo] + m;
    return tl;
}

// Tile table of an offsets vector in shared memory: s_toff[e] = sum over
// e' < e of ceil(count/128), s_toff[E] = row tiles in all. Returns false
// (and sets MOE_DEVERR_BAD_OFFSETS once) when offsets are not monotone from
// 0 to R. Whole block; E <= MOE_MAX_EXPERTS.
__device__ bool block_tile_table(const int32_t* __restrict__ offsets, int E, int R, int* s_off,
                                 int* s_toff, int* s_bad, int* status) {
    const int tid = threadIdx.x, lane = tid & 31;
    for (int e = tid; e <= E; e += blockDim.x) s_off[e] = offsets[e];
    __syncthreads();
    if (tid < 32) {
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
    if (*s_bad && tid == 0 && blockIdx.x == 0) set_status(status, MOE_DEVERR_BAD_OFFSETS);
    return !*s_bad;
}

// Expert whose tile range holds row tile g (s_toff ascending, g < s_toff[E]).
__device__ __forceinline__ int expert_of_tile(const int* s_toff, int E, int g) {
    int lo = 0, hi = E - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_toff[mid] <= g) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

// SWIGLU: B tile = 128 rows of W1 then 128 rows of W3 at the same n0; the
// epilogue writes Hq/Hs (128 output columns per tile). Otherwise B = 256 rows
// of W2 (rows past N read as zeros) and the epilogue writes bf16 Ye (256
// columns, those past N skipped).
template <bool SWIGLU>
__global__ void __launch_bounds__(THREADS, 1)
    mx_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                   const __grid_constant__ CUtensorMap tmB0,
                   const __grid_constant__ CUtensorMap tmB1, const uint8_t* __restrict__ sfAp,
                   const uint8_t* __restrict__ sfBp, const int32_t* __restrict__ offsets, int E, int R,
                   int K, int N, uint8_t* __restrict__ out_q, uint8_t* __restrict__ out_sp,
                   __nv_bfloat16* __restrict__ out_bf16, int64_t ldo, int* status,
                   __nv_bfloat16* __restrict__ save_a, __nv_bfloat16* __restrict__ save_b) {
    constexpr int OUT_N = SWIGLU ? MMA_N / 2 : MMA_N;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sf_smem = smem + STAGES * STAGE_BYTES;
    uint8_t* meta = sf_smem + STAGES * SF_STAGE_BYTES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(meta);
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(meta + NUM_BARS * 8);
    volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
    int* s_bad = reinterpret_cast<int*>(s_tmem + 2);
    int* s_off = reinterpret_cast<int*>(meta + NUM_BARS * 8 + 16);
    int* s_toff = s_off + (MOE_MAX_EXPERTS + 1);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint64_t wl = wait_limit();  // the pipeline waits' time limit, read once

    if (!block_tile_table(offsets, E, R, s_off, s_toff, s_bad, status)) return;
    const int NB = (N + OUT_N - 1) / OUT_N;
    const int total = s_toff[E] * NB;
    if ((int)blockIdx.x >= total) return;
    const int KS = K / BK;  // 128-byte slabs = pipeline stages per tile

    uint64_t* full = bars;
    uint64_t* empty = bars + STAGES;
    uint64_t* tfull = bars + 2 * STAGES;
    uint64_t* tempty = bars + 2 * STAGES + 1;
    uint64_t* drain = bars + 2 * STAGES + 2;
    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(smem_u32(full + s), 1);  // the stage's TMA and bulk bytes
            mbar_init(smem_u32(empty + s), 1);
        }
        mbar_init(smem_u32(tfull), 1);
        mbar_init(smem_u32(tempty), EPI_WARPS);
        mbar_init(smem_u32(drain), 1);
        *s_abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        prefetch_map(&tmA);
        prefetch_map(&tmB0);
        if (SWIGLU) prefetch_map(&tmB1);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(s_tmem), TMEM_ALLOC);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *s_tmem;

    if (warp == 0) {
        // ------------------------------------------------ producer (lane 0)
        int stage = 0;
        uint32_t phase = 0, issued_mask = 0, issued_parity = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
            const Tile tl = decode_tile(t, NB, E, OUT_N, s_toff, s_off);
            for (int kb = 0; kb < KS; ++kb) {
                if (!mbar_wait(smem_u32(empty + stage), phase ^ 1u, s_abort, status, wl)) {
                    ok = false;
                    break;
                }
                const uint32_t fb = smem_u32(full + stage);
                const uint32_t sfs = smem_u32(sf_smem + stage * SF_STAGE_BYTES);
                if (lane == 0) {
                    mbar_expect_tx(fb, (uint32_t)(STAGE_BYTES + 3 * SF_BLOCK));
                    // packed scales of this slab: the A tile's block, then the
                    // B tile's two 128-row blocks
                    bulk_load(sfs, sfAp + ((size_t)tl.tile * KS + kb) * SF_BLOCK, SF_BLOCK, fb);
                    const size_t blk = ((size_t)tl.e * NB + tl.n0 / OUT_N) * KS + kb;
                    bulk_load(sfs + SF_BLOCK, sfBp + blk * (2 * SF_BLOCK), 2u * SF_BLOCK, fb);
                    const int kc = kb * BK;
                    const uint32_t sa = smem_u32(smem + stage * STAGE_BYTES);
                    const uint32_t sb = sa + A_BYTES;
                    tma_load_2d(sa, &tmA, fb, kc, tl.row0);
                    if (SWIGLU) {
                        tma_load_3d(sb, &tmB0, fb, kc, tl.n0, tl.e);
                        tma_load_3d(sb + B_BYTES / 2, &tmB1, fb, kc, tl.n0, tl.e);
                    } else {
                        tma_load_3d(sb, &tmB0, fb, kc, tl.n0, tl.e);
                    }
                }
                issued_mask |= 1u << stage;
                issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
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
    } else if (warp == 1 && lane == 0) {
        // ------------------------------------------------ MMA issuer
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        int i = 0;
        const uint32_t sfa_t = tmem_base + SFA_COL;
        const uint32_t sfb_t = tmem_base + SFB_COL;
        for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++i) {
            // the epilogue has moved the previous tile's accumulator out
            if (!mbar_wait(smem_u32(tempty), ((uint32_t)i & 1u) ^ 1u, s_abort, status,
                           wl)) {
                ok = false;
                break;
            }
            tc_fence_after();
            for (int kb = 0; kb < KS; ++kb) {
                if (!mbar_wait(smem_u32(full + stage), phase, s_abort, status, wl)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t sfs = smem_u32(sf_smem + stage * SF_STAGE_BYTES);
                tmem_cp_sf(sfa_t, sf_desc(sfs));
                tmem_cp_sf(sfb_t, sf_desc(sfs + SF_BLOCK));
                tmem_cp_sf(sfb_t + 4u, sf_desc(sfs + 2 * SF_BLOCK));
                const uint32_t sa = smem_u32(smem + stage * STAGE_BYTES);
                const uint64_t ad = sw128_desc(sa);
                const uint64_t bd = sw128_desc(sa + A_BYTES);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_mx(tmem_base, ad + 2 * ks, bd + 2 * ks, mx_idesc(ks),
                           sfa_t | ((uint32_t)ks << 30), sfb_t | ((uint32_t)ks << 30),
                           (kb | ks) != 0);
                tc_commit(smem_u32(empty + stage));
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (ok) tc_commit(smem_u32(tfull));
        }
        if (!ok) {
            tc_commit(smem_u32(drain));
            volatile int no_abort = 0;
            mbar_wait(smem_u32(drain), 0, &no_abort, nullptr, DRAIN_LIMIT_NS);
        }
    } else if (warp >= 2) {
        // ------------------------------------------------ epilogue: warp w
        // reads TMEM lanes 32 (w % 4)..+31 (its rows) and column half h
        const int q = warp & 3;
        const int h = (warp - 2) >> 2;
        const int r_in_tile = q * 32 + lane;
        int i = 0;
        for (int t = blockIdx.x; t < total; t += gridDim.x, ++i) {
            const Tile tl = decode_tile(t, NB, E, OUT_N, s_toff, s_off);
            if (!mbar_wait(smem_u32(tfull), (uint32_t)i & 1u, s_abort, status, wl))
                break;
            tc_fence_after();
            const uint32_t ta = tmem_base + ((uint32_t)(q * 32) << 16);
            uint32_t acc[128];
            if constexpr (SWIGLU) {
                // W1 columns 64h..64h+63 and the W3 columns 128 further on
                tmem_ld32(ta + 64 * h, acc);
                tmem_ld32(ta + 64 * h + 32, acc + 32);
                tmem_ld32(ta + MMA_N / 2 + 64 * h, acc + 64);
                tmem_ld32(ta + MMA_N / 2 + 64 * h + 32, acc + 96);
            } else {
#pragma unroll
                for (int c = 0; c < 4; ++c) tmem_ld32(ta + 128 * h + 32 * c, acc + 32 * c);
            }
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(tempty));
            const int grow = tl.row0 + r_in_tile;
            const bool valid = grow < tl.row_end;
            const size_t gr = (size_t)(valid ? grow : 0);
            if constexpr (SWIGLU) {
                // H scales go to the tile-packed layout the down GEMM copies
                // (tile rows past the expert's rows get 0)
                const uint32_t sp_word = 16u * (uint32_t)(r_in_tile & 31) + 4u * (uint32_t)(r_in_tile >> 5);
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    const int col = tl.n0 + 64 * h + 32 * c;
                    uint8_t* sp = out_sp + ((size_t)tl.tile * (ldo / BK) + col / BK) * SF_BLOCK +
                                  sp_word + (col / 32) % 4;
                    if (!valid) {
                        *sp = 0;
                        continue;
                    }
                    float v[32];
                    if (save_a != nullptr) {
                        // pre-activations kept (bf16) for the backward pass
                        uint4* da = reinterpret_cast<uint4*>(save_a + gr * ldo + col);
                        uint4* db = reinterpret_cast<uint4*>(save_b + gr * ldo + col);
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
#pragma unroll
                            for (int j = 0; j < 8; ++j) v[j] = __uint_as_float(acc[32 * c + 8 * u + j]);
                            da[u] = pack8(v);
#pragma unroll
                            for (int j = 0; j < 8; ++j)
                                v[j] = __uint_as_float(acc[64 + 32 * c + 8 * u + j]);
                            db[u] = pack8(v);
                        }
                    }
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const float g = __uint_as_float(acc[32 * c + j]);
                        v[j] = g / (1.0f + __expf(-g)) * __uint_as_float(acc[64 + 32 * c + j]);
                    }
                    float sc;
                    const uint8_t sbyte = mxc::e8m0_scale(v, &sc);
                    uint32_t w[8];
                    mxc::encode32_e8m0(v, sbyte, w);
                    uint4* dq = reinterpret_cast<uint4*>(out_q + gr * ldo + col);
                    dq[0] = make_uint4(w[0], w[1], w[2], w[3]);
                    dq[1] = make_uint4(w[4], w[5], w[6], w[7]);
                    *sp = sbyte;
                }
            } else if (valid) {
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int col = tl.n0 + 128 * h + 32 * c;
                    if (col < N) {
                        float v[32];
#pragma unroll
                        for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(acc[32 * c + j]);
                        uint4* d = reinterpret_cast<uint4*>(out_bf16 + gr * ldo + col);
#pragma unroll
                        for (int u = 0; u < 4; ++u) d[u] = pack8(v + 8 * u);
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) {
        __syncwarp();
        tmem_dealloc(tmem_base, TMEM_ALLOC);
    }
}

// Quantise each token row once (blocks of 32 along d, UE8M0 scales) and
// write the codes and scales to its k slots. One thread per 32-value block.
__global__ void __launch_bounds__(256) mx_dispatch_kernel(const __nv_bfloat16* __restrict__ x,
                                                          const int32_t* __restrict__ slot, int T,
                                                          int d, int k, int64_t R,
                                                          uint8_t* __restrict__ Xq,
                                                          uint8_t* __restrict__ Xs, int* status) {
    const int bpr = d / 32;
    const int64_t n = (int64_t)T * bpr;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int t = (int)(i / bpr);
        const int b = (int)(i - (int64_t)t * bpr);
        float v[32];
        const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * d + b * 32);
#pragma unroll
        for (int u = 0; u < 4; ++u) unpack8(__ldcs(src + u), v + 8 * u);
        float sc;
        const uint8_t sbyte = mxc::e8m0_scale(v, &sc);
        uint32_t w[8];
        mxc::encode32_e8m0(v, sbyte, w);
        const uint4 c0 = make_uint4(w[0], w[1], w[2], w[3]);
        const uint4 c1 = make_uint4(w[4], w[5], w[6], w[7]);
        for (int j = 0; j < k; ++j) {
            const int s = slot[(size_t)t * k + j];
            if (s < 0 || s >= R) {
                set_status(status, MOE_DEVERR_BAD_INDEX);
                continue;
            }
            uint4* dq = reinterpret_cast<uint4*>(Xq + (size_t)s * d + b * 32);
            dq[0] = c0;
            dq[1] = c1;
            Xs[(size_t)s * bpr + b] = sbyte;
        }
    }
}

// Weight scales packed for the tensor-core scale copy. For every expert,
// 256-row B tile of the kernel (gate/up: rows n0..n0+127 of W1 then of W3,
// n0 = 128 nb; down: rows n0..n0+255 of W2, n0 = 256 nb, rows past the
// matrix zero) and 128-element K slab s, two 512-byte blocks (tile rows
// 0..127, then 128..255) each hold the four scale bytes of their 128 rows in
// the 32-row x 16-byte order tcgen05.cp.32x128b.warpx4 copies: row m's word
// at 16 (m % 32) + 4 (m / 32). Blocks are ordered (expert, n-block, slab,
// half), so one stage's blocks are adjacent. One thread per word.
__global__ void __launch_bounds__(256)
    pack_scales_kernel(const uint8_t* __restrict__ Sa, const uint8_t* __restrict__ Sb,
                       int64_t rows_per_expert, int64_t sf_row, int nb_count, int ks_count,
                       int64_t n_words, uint32_t* __restrict__ packed) {
    for (int64_t w = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; w < n_words;
         w += (int64_t)gridDim.x * blockDim.x) {
        const int64_t blk = w >> 7;          // 128 words per 512-byte block
        const int pos = (int)(w & 127);      // word position in the block
        const int m = (pos >> 2) + 32 * (pos & 3);  // row within the block
        const int half = (int)(blk & 1);
        const int64_t bs = blk >> 1;
        const int slab = (int)(bs % ks_count);
        const int64_t eb = bs / ks_count;
        const int nb = (int)(eb % nb_count);
        const int64_t e = eb / nb_count;
        const uint8_t* src;
        int64_t row;
        if (Sb != nullptr) {  // gate/up: the W1 block, then the W3 block
            src = half ? Sb : Sa;
            row = (int64_t)nb * 128 + m;
        } else {
            src = Sa;
            row = (int64_t)nb * 256 + half * 128 + m;
        }
        uint32_t word = 0;
        if (row < rows_per_expert) {
            const uint8_t* p = src + (e * rows_per_expert + row) * sf_row + 4 * slab;
            word = (uint32_t)p[0] | ((uint32_t)p[1] << 8) | ((uint32_t)p[2] << 16) |
                   ((uint32_t)p[3] << 24);
        }
        packed[w] = word;
    }
}

// Activation scales between rows ([R, K/32] bytes) and the tile-packed
// layout the GEMMs copy: for every row tile g of the expert-sorted rows
// (experts in order, ceil(count/128) tiles each) and 128-element K slab s, a
// 512-byte block holds the word (four K-block bytes) of tile row m at
// 16 (m % 32) + 4 (m / 32); blocks ordered (tile, slab); tile rows past the
// expert's rows hold 0. This kernel: one thread per word (unpack uses it;
// pack uses act_scales_pack_kernel below).
template <bool UNPACK>
__global__ void __launch_bounds__(256)
    act_scales_kernel(const int32_t* __restrict__ offsets, int E, int R, int ks_count,
                      int64_t n_words, const uint32_t* __restrict__ src,
                      uint32_t* __restrict__ dst, int* status) {
    __shared__ int s_off[MOE_MAX_EXPERTS + 1];
    __shared__ int s_toff[MOE_MAX_EXPERTS + 1];
    __shared__ int s_bad;
    if (!block_tile_table(offsets, E, R, s_off, s_toff, &s_bad, status)) return;
    const int64_t used = (int64_t)s_toff[E] * ks_count * 128;
    for (int64_t w = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; w < n_words;
         w += (int64_t)gridDim.x * blockDim.x) {
        if (w >= used) break;  // tiles past the table's end are not used
        const int pos = (int)(w & 127);
        const int64_t blk = w >> 7;
        const int slab = (int)(blk % ks_count);
        const int g = (int)(blk / ks_count);
        const int m = (pos >> 2) + 32 * (pos & 3);
        const int e = expert_of_tile(s_toff, E, g);
        const int row = s_off[e] + (g - s_toff[e]) * BM + m;
        const bool in = row < s_off[e + 1];
        const int64_t rw = (int64_t)row * ks_count + slab;  // row-layout word
        if (UNPACK) {
            if (in) dst[rw] = src[w];
        } else {
            dst[w] = in ? src[rw] : 0u;
        }
    }
}

// Packing, one CTA per row tile at a time (grid stride): the tile's 128 rows
// x up to 32 slab words are read row by row (coalesced), held slab-major in
// shared memory, and written block by block (coalesced 512-byte blocks).
// Row m of a slab sits at m + 8 (m / 32) in its shared row (pitch 153
// words), so both the column writes and the block-order reads hit 32
// different banks.
constexpr int PK_SLABS = 32;
constexpr int PK_PITCH = 153;

__global__ void __launch_bounds__(256)
    act_scales_pack_kernel(const int32_t* __restrict__ offsets, int E, int R, int ks_count,
                           const uint32_t* __restrict__ src, uint32_t* __restrict__ dst,
                           int* status) {
    __shared__ int s_off[MOE_MAX_EXPERTS + 1];
    __shared__ int s_toff[MOE_MAX_EXPERTS + 1];
    __shared__ int s_bad;
    __shared__ uint32_t tile[PK_SLABS * PK_PITCH];
    if (!block_tile_table(offsets, E, R, s_off, s_toff, &s_bad, status)) return;
    const int tid = threadIdx.x;
    const int ntiles = s_toff[E];
    for (int g = blockIdx.x; g < ntiles; g += gridDim.x) {
        const int e = expert_of_tile(s_toff, E, g);
        const int row0 = s_off[e] + (g - s_toff[e]) * BM;
        const int rend = s_off[e + 1];
        for (int sc = 0; sc < ks_count; sc += PK_SLABS) {
            const int nsl = ks_count - sc < PK_SLABS ? ks_count - sc : PK_SLABS;
            __syncthreads();  // the previous chunk's words have been written out
            for (int i = tid; i < BM * nsl; i += blockDim.x) {
                const int r = i / nsl, j = i - r * nsl;
                const int row = row0 + r;
                tile[j * PK_PITCH + r + 8 * (r >> 5)] =
                    row < rend ? src[(int64_t)row * ks_count + sc + j] : 0u;
            }
            __syncthreads();
            for (int i = tid; i < nsl * BM; i += blockDim.x) {
                const int j = i >> 7, pos = i & 127;
                const int m = (pos >> 2) + 32 * (pos & 3);
                dst[((int64_t)g * ks_count + sc + j) * BM + pos] =
                    tile[j * PK_PITCH + m + 8 * (m >> 5)];
            }
        }
    }
}

template <bool SWIGLU>
static int launch(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                  const uint8_t* sfA, const uint8_t* sfBp, const int32_t* offsets, int64_t E, int64_t R, int64_t K, int64_t N, uint8_t* oq,
                  uint8_t* os, __nv_bfloat16* ob, int64_t ldo, cudaStream_t st,
                  void* save_a = nullptr, void* save_b = nullptr) {
    auto kern = mx_gemm_kernel<SWIGLU>;
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
    const int out_n = SWIGLU ? MMA_N / 2 : MMA_N;
    const int64_t max_tiles = (R / BM + E) * ((N + out_n - 1) / out_n);
    const int64_t sms = num_sms();
    const int grid = (int)(max_tiles < sms ? max_tiles : sms);
    if (grid <= 0) return MOE_OK;
    kern<<<grid, THREADS, SMEM_BYTES, st>>>(a, b0, b1, sfA, sfBp, offsets, (int)E,
                                           (int)R, (int)K, (int)N, oq, os, ob, ldo, status_ptr(),
                                           static_cast<__nv_bfloat16*>(save_a),
                                           static_cast<__nv_bfloat16*>(save_b));
    return launch_status();
}

constexpr CUtensorMapDataType U8 = CU_TENSOR_MAP_DATA_TYPE_UINT8;

}  // namespace mxg
}  // namespace moe

using namespace moe;
using namespace moe::tc;

extern "C" int moe_dispatch_mxfp8(const void* x, const int32_t* slot, int64_t T, int64_t d, int k,
                                  uint8_t* Xq, uint8_t* Xs, void* stream) {
    if (T < 0 || d <= 0 || d % 32 != 0 || k < 1 || k > MOE_MAX_TOPK) return MOE_ERR_INVALID;
    if (T == 0) return MOE_OK;
    if (!x || !slot || !Xq || !Xs || !aligned16(x) || !aligned16(Xq)) return MOE_ERR_INVALID;
    if (T * k > INT32_MAX) return MOE_ERR_UNSUPPORTED;
    if (check_only()) return MOE_OK;
    const int64_t n = T * (d / 32);
    int64_t g = (n + 255) / 256;
    const int64_t cap = (int64_t)num_sms() * 16;
    if (g > cap) g = cap;
    mxg::mx_dispatch_kernel<<<(int)g, 256, 0, as_stream(stream)>>>(
        static_cast<const __nv_bfloat16*>(x), slot, (int)T, (int)d, k, T * k, Xq, Xs, status_ptr());
    return launch_status();
}

static int mx_check(const void* A, const void* As, const void* B, const void* Bp,
                    const int32_t* offsets, int64_t E, int64_t R, int64_t d, int64_t F) {
    if (E < 1 || E > MOE_MAX_EXPERTS || R < 0 || d <= 0 || F <= 0) return MOE_ERR_INVALID;
    if (d % 128 != 0 || F % 128 != 0) return MOE_ERR_UNSUPPORTED;
    if (R > INT32_MAX - 2 * mxg::BM || d > (1 << 24) || F > (1 << 24)) return MOE_ERR_UNSUPPORTED;
    if (!offsets || !A || !As || !B || !Bp) return MOE_ERR_INVALID;
    if (!aligned16(A) || !aligned16(B) || !aligned16(Bp) || !aligned16(As)) return MOE_ERR_INVALID;
    return MOE_OK;
}

extern "C" int mxfp8_pack_weight_scales(const uint8_t* W1s, const uint8_t* W3s,
                                        const uint8_t* W2s, int64_t E, int64_t d, int64_t F,
                                        uint8_t* Ps13, uint8_t* Ps2, void* stream) {
    if (E < 1 || E > MOE_MAX_EXPERTS || d <= 0 || F <= 0) return MOE_ERR_INVALID;
    if (d % 128 != 0 || F % 128 != 0) return MOE_ERR_UNSUPPORTED;
    if ((W1s == nullptr) != (W3s == nullptr) || (W1s == nullptr) != (Ps13 == nullptr))
        return MOE_ERR_INVALID;
    if ((W2s == nullptr) != (Ps2 == nullptr)) return MOE_ERR_INVALID;
    if ((Ps13 && !aligned16(Ps13)) || (Ps2 && !aligned16(Ps2))) return MOE_ERR_INVALID;
    if (check_only()) return MOE_OK;
    cudaStream_t st = as_stream(stream);
    const int64_t cap = (int64_t)num_sms() * 8;
    if (Ps13) {  // gate/up tiles: 128 rows of W1 + 128 of W3 per n-block, K = d
        const int nb = (int)(F / 128), ks = (int)(d / 128);
        const int64_t words = E * nb * ks * 2 * 128;
        int64_t g = (words + 255) / 256;
        if (g > cap) g = cap;
        mxg::pack_scales_kernel<<<(int)g, 256, 0, st>>>(W1s, W3s, F, d / 32, nb, ks, words,
                                                       reinterpret_cast<uint32_t*>(Ps13));
    }
    if (Ps2) {   // down tiles: 256 rows of W2 per n-block, K = F
        const int nb = (int)((d + 255) / 256), ks = (int)(F / 128);
        const int64_t words = E * nb * ks * 2 * 128;
        int64_t g = (words + 255) / 256;
        if (g > cap) g = cap;
        mxg::pack_scales_kernel<<<(int)g, 256, 0, st>>>(W2s, nullptr, d, F / 32, nb, ks, words,
                                                       reinterpret_cast<uint32_t*>(Ps2));
    }
    return launch_status();
}

static int act_scales(const uint8_t* src, const int32_t* offsets, int64_t E, int64_t R,
                      int64_t K, uint8_t* dst, void* stream, bool unpack) {
    if (E < 1 || E > MOE_MAX_EXPERTS || R < 0 || K <= 0) return MOE_ERR_INVALID;
    if (K % 128 != 0) return MOE_ERR_UNSUPPORTED;
    if (R > INT32_MAX - 2 * mxg::BM) return MOE_ERR_UNSUPPORTED;
    if (R == 0) return MOE_OK;
    if (!src || !dst || !offsets) return MOE_ERR_INVALID;
    if (!aligned16(src) || !aligned16(dst)) return MOE_ERR_INVALID;
    if (check_only()) return MOE_OK;
    const int ks = (int)(K / 128);
    const int64_t words = (R / mxg::BM + E) * ks * 128;
    // about one word per thread: each word is a dependent load and store
    int64_t g = (words + 255) / 256;
    const int64_t cap = (int64_t)num_sms() * 32;
    if (g > cap) g = cap;
    const uint32_t* s = reinterpret_cast<const uint32_t*>(src);
    uint32_t* d = reinterpret_cast<uint32_t*>(dst);
    if (unpack) {
        mxg::act_scales_kernel<true><<<(int)g, 256, 0, as_stream(stream)>>>(
            offsets, (int)E, (int)R, ks, words, s, d, status_ptr());
    } else {
        int64_t tiles = R / mxg::BM + E;
        const int64_t tcap = (int64_t)num_sms() * 4;
        if (tiles > tcap) tiles = tcap;
        mxg::act_scales_pack_kernel<<<(int)tiles, 256, 0, as_stream(stream)>>>(
            offsets, (int)E, (int)R, ks, s, d, status_ptr());
    }
    return launch_status();
}

extern "C" size_t mxfp8_act_scales_packed_size(int64_t E, int64_t R, int64_t K) {
    if (E < 1 || R < 0 || K <= 0 || K % 128 != 0) return 0;
    return (size_t)(R / mxg::BM + E) * (size_t)(K / 128) * mxg::SF_BLOCK;
}

extern "C" int mxfp8_pack_act_scales(const uint8_t* S, const int32_t* offsets, int64_t E,
                                     int64_t R, int64_t K, uint8_t* Sp, void* stream) {
    return act_scales(S, offsets, E, R, K, Sp, stream, false);
}

extern "C" int mxfp8_unpack_act_scales(const uint8_t* Sp, const int32_t* offsets, int64_t E,
                                       int64_t R, int64_t K, uint8_t* S, void* stream) {
    return act_scales(Sp, offsets, E, R, K, S, stream, true);
}

extern "C" int moe_grouped_gate_up_mxfp8_save(const uint8_t* Xq, const uint8_t* Xs,
                                              const uint8_t* W1q, const uint8_t* W3q,
                                              const uint8_t* Ps13, int64_t w13_expert_stride,
                                              const int32_t* offsets, int64_t E, int64_t R,
                                              int64_t d, int64_t F, uint8_t* Hq, uint8_t* Hs,
                                              void* A_out, void* B_out, void* stream) {
    int rc = mx_check(Xq, Xs, W1q, Ps13, offsets, E, R, d, F);
    if (rc != MOE_OK) return rc;
    if (!W3q || !Hq || !Hs || !aligned16(W3q) || !aligned16(Hq) || !aligned16(Hs))
        return MOE_ERR_INVALID;
    if ((A_out == nullptr) != (B_out == nullptr)) return MOE_ERR_INVALID;
    if (A_out && (!aligned16(A_out) || !aligned16(B_out))) return MOE_ERR_INVALID;
    if ((w13_expert_stride < F * d && E > 1) || w13_expert_stride % 128 != 0) return MOE_ERR_INVALID;
    if (R == 0) return MOE_OK;
    CUtensorMap a, b0, b1;
    if (!make_map_2d(&a, Xq, mxg::U8, 1, d, R, mxg::BM) ||
        !make_map_3d(&b0, W1q, mxg::U8, 1, d, F, E, w13_expert_stride, mxg::MMA_N / 2) ||
        !make_map_3d(&b1, W3q, mxg::U8, 1, d, F, E, w13_expert_stride, mxg::MMA_N / 2))
        return MOE_ERR_CUDA;
    return mxg::launch<true>(a, b0, b1, Xs, Ps13, offsets, E, R, d, F, Hq, Hs, nullptr, F,
                             as_stream(stream), A_out, B_out);
}

extern "C" int moe_grouped_gate_up_mxfp8(const uint8_t* Xq, const uint8_t* Xs, const uint8_t* W1q,
                                         const uint8_t* W3q, const uint8_t* Ps13,
                                         int64_t w13_expert_stride, const int32_t* offsets,
                                         int64_t E, int64_t R, int64_t d, int64_t F, uint8_t* Hq,
                                         uint8_t* Hs, void* stream) {
    return moe_grouped_gate_up_mxfp8_save(Xq, Xs, W1q, W3q, Ps13, w13_expert_stride, offsets, E,
                                          R, d, F, Hq, Hs, nullptr, nullptr, stream);
}

extern "C" int moe_grouped_down_mxfp8(const uint8_t* Hq, const uint8_t* Hs, const uint8_t* W2q,
                                      const uint8_t* Ps2, int64_t w2_expert_stride,
                                      const int32_t* offsets, int64_t E, int64_t R, int64_t d,
                                      int64_t F, void* Ye, void* stream) {
    int rc = mx_check(Hq, Hs, W2q, Ps2, offsets, E, R, d, F);
    if (rc != MOE_OK) return rc;
    if (!Ye || !aligned16(Ye)) return MOE_ERR_INVALID;
    if ((w2_expert_stride < F * d && E > 1) || w2_expert_stride % 128 != 0) return MOE_ERR_INVALID;
    if (R == 0) return MOE_OK;
    CUtensorMap a, b0;
    if (!make_map_2d(&a, Hq, mxg::U8, 1, F, R, mxg::BM) ||
        !make_map_3d(&b0, W2q, mxg::U8, 1, F, d, E, w2_expert_stride, mxg::MMA_N))
        return MOE_ERR_CUDA;
    return mxg::launch<false>(a, b0, b0, Hs, Ps2, offsets, E, R, F, d, nullptr, nullptr,
                              static_cast<__nv_bfloat16*>(Ye), d, as_stream(stream));
}
