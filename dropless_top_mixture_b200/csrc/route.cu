// Route step of the dropless top-k MoE layer on sm_100a.
//
//   a0  router logits  logits[t,e] = sum_j x[t,j]*Wr[e,j]: bf16 on the tensor
//                      cores (fp32 accumulation); fp32 as four fmaf chains
//                      over the quarters of j, added in order
//   a1  fp32 softmax + top-k (ties to the lower expert index)
//   a2  routing metadata: counts, offsets, slots, tile offsets
//
// "Transformers 中的 OLMoE" (blog.gitcode.com) §2: softmax over the expert
// logits in fp32, then top-k, optional renormalisation; bias-free (E, d)
// router weight. "olmoforge" README, capability table: the routing table is
// built and kept on the device, so nothing is copied back to the host.
//
// Routing metadata is a stable counting sort of the token-major (t, j) list
// by expert, built in three launches:
//   1. topk_group: one CTA per chunk of 8 to 32 consecutive tokens (a group
//      of 1 to 16 lanes per token, by E). It selects the k experts of each
//      token in order, marks each selection in a per-expert bit mask over the
//      chunk's tokens, and reads a token's rank among the chunk's rows of the
//      expert (stable by token) off the mask. Per-chunk counts go to
//      ws_count[e][c]. For the fp32 router it also adds the four quarter
//      planes (and writes the logits out if asked).
//   2. scan: one block per expert scans ws_count[e][:] over chunks (exclusive,
//      in place) and writes counts[e]; the last block to finish (ticket
//      counter) scans counts into offsets and tile_offsets.
//   3. finalize: slot = offsets[e] + chunk_base[e][c] + rank.
// Integer work only after the top-k, so the result is bit-exact and
// independent of scheduling.
#include "tc_sm100.cuh"

namespace moe {
namespace route {

constexpr int LOGIT_TT = 64;       // tokens per router-logits tile
constexpr int LOGIT_TE = 64;       // experts per router-logits tile
constexpr int LOGIT_TK = 16;       // contraction chunk staged in shared memory
constexpr int LOGIT_LD = 68;       // padded row of the staged chunk (floats)
constexpr int LOGIT_D_ALIGN = 128; // d must be a multiple of this

// ------------------------------------------------------------------ a0

// 16-byte asynchronous copy global -> shared; src_bytes = 0 fills zeros.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, int src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
                 "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.wait_group 0;" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait_one() {  // all but the newest group
    asm volatile("cp.async.wait_group 1;" ::: "memory");
}

// 16 consecutive fp32 elements of a row landed in shared memory, to registers.
__device__ __forceinline__ void landed16_to_f32(const uint4* p, float* f) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float4 v = reinterpret_cast<const float4*>(p)[i];
        f[4 * i] = v.x; f[4 * i + 1] = v.y; f[4 * i + 2] = v.z; f[4 * i + 3] = v.w;
    }
}

// fp32 router. The logit of (t, e) is four fmaf chains, one per contiguous
// quarter of j, each from +0.0 in ascending j, their sums added in order
// ((c0 + c1) + c2) + c3. One CTA (64 threads) computes one quarter's chains
// for a 64-token x 64-expert tile (grid z = quarter) and writes them to that
// quarter's plane; the top-k kernel adds the four planes in order. Eight
// CTAs are resident per SM (127 registers).
//   staging: thread i copies 16 consecutive elements of x row t0 + i and of
//            Wr row e0 + i per chunk into its own landing slots with
//            cp.async (one chunk ahead), then stores them k-major into shared
//            memory (a warp writes 32 consecutive floats of one k: no
//            conflicts);
//   compute: thread (ty, tx) = (i / 8, i % 8) owns tokens 4ty..4ty+3 and
//            32+4ty..32+4ty+3 and experts 4tx..4tx+3 and 32+4tx..32+4tx+3:
//            64 accumulators; per k, 4 shared float4 loads (the eight tx of a
//            phase read 128 consecutive bytes) feed 64 FMAs.
constexpr int LOGIT_THREADS = 64;
constexpr int LOGIT_SPLIT = 4;  // quarter chains per logit

__global__ void __launch_bounds__(LOGIT_THREADS, 8) router_logits_kernel(
    const float* __restrict__ x, const float* __restrict__ Wr, int T, int d, int E,
    float* __restrict__ planes, int64_t pstride) {
    constexpr int PIECES = LOGIT_TK * (int)sizeof(float) / 16;  // 16-byte pieces per row chunk
    constexpr int PEL = 16 / (int)sizeof(float);                // elements per piece
    __shared__ __align__(16) float xs[2][LOGIT_TK][LOGIT_LD];
    __shared__ __align__(16) float ws[2][LOGIT_TK][LOGIT_LD];
    __shared__ __align__(16) uint4 land[2][LOGIT_THREADS][PIECES];  // [x | Wr][row][piece]
    const int tid = threadIdx.x;
    const int t0 = blockIdx.x * LOGIT_TT;
    const int e0 = blockIdx.y * LOGIT_TE;
    const int dq = d / LOGIT_SPLIT;
    const int kbeg = blockIdx.z * dq;
    float* __restrict__ logits = planes + (size_t)blockIdx.z * pstride;
    const bool xok = (t0 + tid) < T;
    const bool wok = (e0 + tid) < E;
    // rows past T or E are zero-filled; their source address stays row 0's
    const float* xp = x + (size_t)(xok ? t0 + tid : 0) * d + kbeg;
    const float* wp = Wr + (size_t)(wok ? e0 + tid : 0) * d + kbeg;
    const uint32_t lx = (uint32_t)__cvta_generic_to_shared(&land[0][tid][0]);
    const uint32_t lw = (uint32_t)__cvta_generic_to_shared(&land[1][tid][0]);
    const int ty = tid >> 3, tx = tid & 7;
    float acc[8][8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

#pragma unroll
    for (int p = 0; p < PIECES; ++p) {
        cp_async16(lx + 16 * p, xp + p * PEL, xok ? 16 : 0);
        cp_async16(lw + 16 * p, wp + p * PEL, wok ? 16 : 0);
    }
    cp_async_commit();
    int buf = 0;
    for (int k0 = 0; k0 < dq; k0 += LOGIT_TK, buf ^= 1) {
        cp_async_wait_all();  // this thread's own copies of chunk k0
        {
            float f[16];
            landed16_to_f32(&land[0][tid][0], f);
#pragma unroll
            for (int i = 0; i < 16; ++i) xs[buf][i][tid] = f[i];
            landed16_to_f32(&land[1][tid][0], f);
#pragma unroll
            for (int i = 0; i < 16; ++i) ws[buf][i][tid] = f[i];
        }
        __syncthreads();
        if (k0 + LOGIT_TK < dq) {
#pragma unroll
            for (int p = 0; p < PIECES; ++p) {
                cp_async16(lx + 16 * p, xp + k0 + LOGIT_TK + p * PEL, xok ? 16 : 0);
                cp_async16(lw + 16 * p, wp + k0 + LOGIT_TK + p * PEL, wok ? 16 : 0);
            }
            cp_async_commit();
        }
#pragma unroll
        for (int kk = 0; kk < LOGIT_TK; ++kk) {
            const float4 a0 = *reinterpret_cast<const float4*>(&xs[buf][kk][4 * ty]);
            const float4 a1 = *reinterpret_cast<const float4*>(&xs[buf][kk][32 + 4 * ty]);
            const float4 b0 = *reinterpret_cast<const float4*>(&ws[buf][kk][4 * tx]);
            const float4 b1 = *reinterpret_cast<const float4*>(&ws[buf][kk][32 + 4 * tx]);
            const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
        }
        // no second barrier: the next chunk goes to the other buffer, and the
        // barrier after that write keeps any thread from overwriting this
        // buffer before every thread has finished reading it
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int t = t0 + (i < 4 ? 4 * ty + i : 32 + 4 * ty + (i - 4));
        if (t >= T) continue;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int e = e0 + 32 * h + 4 * tx;
            const float* a = &acc[i][4 * h];
            if (e + 3 < E && (E & 3) == 0) {
                *reinterpret_cast<float4*>(&logits[(size_t)t * E + e]) =
                    make_float4(a[0], a[1], a[2], a[3]);
            } else {
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    if (e + j < E) logits[(size_t)t * E + e + j] = a[j];
            }
        }
    }
}

// ------------------------------------------------------------------ a0, bf16
//
// bf16 router: logits = x Wrᵀ on the tensor cores. The pages' router is a
// bias-free linear layer in the model's dtype ("Transformers 中的 OLMoE" §2);
// every bf16 x bf16 product is exact in fp32 and tcgen05 (kind::f16) sums
// them into an fp32 TMEM accumulator, in the order the tensor core chooses.
// One CTA computes a 128-token x EN-expert tile (EN = 64, 128 or 256 from E;
// grid.y covers E > 256): warp 0 lane 0 streams 128-byte K slabs of x and Wr
// with TMA through an RT_STAGES ring, warp 1 lane 0 issues 4 MMAs per slab,
// warps 2..5 read the accumulator (one TMEM lane quarter each) and store fp32
// rows, masked to T and E. Every wait is bounded as in the grouped GEMMs.
//
// While the slabs sit in shared memory the four epilogue warps also sum the
// squares of their rows: thread r of the A tile gives ||x_t||^2 for token
// m0 + r (CTAs with blockIdx.y == 0), and in CTAs with blockIdx.x == 0 the
// B tile's rows give ||w_e||^2. Each is an fp32 sum of exact squares in
// ascending j, so it is at most d 2^-24 (relatively) below the true value;
// the refinement below turns them into a bound on the logit error. A stage
// is free again once the MMAs (one commit) and the four epilogue warps (one
// arrival each) are done with it.
constexpr int RT_BM = 128;
constexpr int RT_THREADS = 192;

template <int EN>
struct RtCfg {
    static constexpr int A_BYTES = RT_BM * 128;
    static constexpr int B_BYTES = EN * 128;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int STAGES = EN <= 128 ? 6 : 4;
    static constexpr int NUM_BARS = 2 * STAGES + 2;
    static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + NUM_BARS * 8 + 16;
    static constexpr uint32_t IDESC = tc::make_idesc(1u, RT_BM, EN);
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
};

template <int EN>
__global__ void __launch_bounds__(RT_THREADS, 1)
    router_logits_tc_kernel(const __grid_constant__ CUtensorMap tmX,
                            const __grid_constant__ CUtensorMap tmW, int T, int d, int E,
                            float* __restrict__ logits, int vec, float* __restrict__ xnorm2,
                            float* __restrict__ wnorm2, int* status) {
    using namespace tc;
    using C = RtCfg<EN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES);
    uint64_t* full = bars;
    uint64_t* empty = bars + C::STAGES;
    uint64_t* done = bars + 2 * C::STAGES;
    uint64_t* drain = done + 1;
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bars + C::NUM_BARS);
    volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint64_t wl = wait_limit();  // the pipeline waits' time limit, read once
    const int m0 = blockIdx.x * RT_BM;
    const int n0 = blockIdx.y * EN;
    const int KS = d / 64;  // 128-byte slabs of bf16

    if (tid == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(smem_u32(full + s), 1);
            mbar_init(smem_u32(empty + s), 1 + 4);  // MMA commit + 4 epilogue warps
        }
        mbar_init(smem_u32(done), 1);
        mbar_init(smem_u32(drain), 1);
        *s_abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        prefetch_map(&tmX);
        prefetch_map(&tmW);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(s_tmem), EN);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *s_tmem;

    if (warp == 0 && lane == 0) {
        // ------------------------------------------------ producer
        int stage = 0;
        uint32_t phase = 0, issued_mask = 0, issued_parity = 0;
        bool ok = true;
        for (int kb = 0; kb < KS; ++kb) {
            if (!mbar_wait(smem_u32(empty + stage), phase ^ 1u, s_abort, status, wl)) {
                ok = false;
                break;
            }
            const uint32_t fb = smem_u32(full + stage);
            const uint32_t sa = smem_u32(smem + stage * C::STAGE_BYTES);
            mbar_expect_tx(fb, (uint32_t)C::STAGE_BYTES);
            tma_load_2d(sa, &tmX, fb, kb * 64, m0);
            tma_load_2d(sa + C::A_BYTES, &tmW, fb, kb * 64, n0);
            issued_mask |= 1u << stage;
            issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
            if (++stage == C::STAGES) {
                stage = 0;
                phase ^= 1u;
            }
        }
        if (!ok) {  // no copy may still be landing when the CTA leaves
            for (int s = 0; s < C::STAGES; ++s)
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
        for (int kb = 0; kb < KS; ++kb) {
            if (!mbar_wait(smem_u32(full + stage), phase, s_abort, status, wl)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t sa = smem_u32(smem + stage * C::STAGE_BYTES);
            const uint64_t ad = sw128_desc(sa);
            const uint64_t bd = sw128_desc(sa + C::A_BYTES);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                tc_mma<false>(tmem_base, ad + 2 * ks, bd + 2 * ks, C::IDESC, (kb | ks) != 0);
            tc_commit(smem_u32(empty + stage));
            if (++stage == C::STAGES) {
                stage = 0;
                phase ^= 1u;
            }
        }
        if (ok) {
            tc_commit(smem_u32(done));
        } else {
            tc_commit(smem_u32(drain));
            volatile int no_abort = 0;
            mbar_wait(smem_u32(drain), 0, &no_abort, nullptr, DRAIN_LIMIT_NS);
        }
    } else if (warp >= 2) {
        // ------------------------------------------------ epilogue
        const int q = warp & 3;
        const int r = q * 32 + lane;           // A row (token m0 + r)
        const int er = (warp - 2) * 32 + lane;  // B rows er and er + 128
        const bool do_x = blockIdx.y == 0, do_w = blockIdx.x == 0;
        float sx = 0.f, sw0 = 0.f, sw1 = 0.f;
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int kb = 0; kb < KS; ++kb) {
            if (!mbar_wait(smem_u32(full + stage), phase, s_abort, status, wl)) {
                ok = false;
                break;
            }
            const uint8_t* st_base = smem + stage * C::STAGE_BYTES;
            // 128-byte rows with the 128-byte swizzle: logical 16-byte chunk c
            // of row r sits at chunk c ^ (r & 7); the chunks are read in
            // logical order, so the sums run in ascending j
            if (do_x) {
                const uint8_t* rowp = st_base + r * 128;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    float f[8];
                    unpack8(*reinterpret_cast<const uint4*>(rowp + 16 * (c ^ (r & 7))), f);
#pragma unroll
                    for (int i = 0; i < 8; ++i) sx = fmaf(f[i], f[i], sx);
                }
            }
            if (do_w) {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int br = er + 128 * h;
                    if (br < EN) {
                        const uint8_t* rowp = st_base + C::A_BYTES + br * 128;
                        float acc = h ? sw1 : sw0;
#pragma unroll
                        for (int c = 0; c < 8; ++c) {
                            float f[8];
                            unpack8(*reinterpret_cast<const uint4*>(rowp + 16 * (c ^ (br & 7))), f);
#pragma unroll
                            for (int i = 0; i < 8; ++i) acc = fmaf(f[i], f[i], acc);
                        }
                        if (h) sw1 = acc; else sw0 = acc;
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(empty + stage));
            if (++stage == C::STAGES) {
                stage = 0;
                phase ^= 1u;
            }
        }
        if (ok) {
            if (do_x && m0 + r < T) xnorm2[m0 + r] = sx;
            if (do_w) {
                if (er < EN && n0 + er < E) wnorm2[n0 + er] = sw0;
                if (er + 128 < EN && n0 + er + 128 < E) wnorm2[n0 + er + 128] = sw1;
            }
        }
        if (ok && mbar_wait(smem_u32(done), 0, s_abort, status, wl)) {
            tc_fence_after();
            const int t = m0 + q * 32 + lane;
            const uint32_t ta = tmem_base + ((uint32_t)(q * 32) << 16);
#pragma unroll 1
            for (int c = 0; c < EN / 32; ++c) {
                uint32_t a[32];
                tmem_ld32(ta + 32 * c, a);
                tmem_wait_ld();
                const int e0 = n0 + 32 * c;
                if (t < T && e0 < E) {
                    float* row = logits + (size_t)t * E + e0;
                    if (vec && e0 + 32 <= E) {
#pragma unroll
                        for (int j = 0; j < 32; j += 4)
                            *reinterpret_cast<float4*>(row + j) =
                                make_float4(__uint_as_float(a[j]), __uint_as_float(a[j + 1]),
                                            __uint_as_float(a[j + 2]), __uint_as_float(a[j + 3]));
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            if (e0 + j < E) row[j] = __uint_as_float(a[j]);
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
        tmem_dealloc(tmem_base, EN);
    }
}

template <int EN>
static int launch_router_tc(const void* x, const void* Wr, int64_t T, int64_t d, int64_t E,
                            float* logits, float* xnorm2, float* wnorm2, cudaStream_t st) {
    using C = RtCfg<EN>;
    auto kern = router_logits_tc_kernel<EN>;
    static bool attr_done[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_done[dev]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 C::SMEM_BYTES) != cudaSuccess)
            return MOE_ERR_CUDA;
        attr_done[dev] = true;
    }
    CUtensorMap mx, mw;
    if (!tc::make_map_2d(&mx, x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d, T, RT_BM) ||
        !tc::make_map_2d(&mw, Wr, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d, E, EN))
        return MOE_ERR_CUDA;
    const int vec = (E % 4 == 0) && aligned16(logits);
    dim3 grid((unsigned)((T + RT_BM - 1) / RT_BM), (unsigned)((E + EN - 1) / EN));
    kern<<<grid, RT_THREADS, C::SMEM_BYTES, st>>>(mx, mw, (int)T, (int)d, (int)E, logits, vec,
                                                  xnorm2, wnorm2, status_ptr());
    return MOE_OK;
}

// ------------------------------------------------------------------ a0, bf16: decisions in the fixed order
//
// The top-k must select exactly what it selects on the fixed-order logits f
// (four fmaf chains over the quarters of j, added in order, as for the fp32
// router). The tensor-core logit v of (t, e) and f are both fp32 sums of the
// same d exact products, in different orders, so they differ by at most
//     B_t = 2 d 2^-23 ||x_t|| max_e ||w_e||.
// Reasoning: with P = sum_j |x_j w_j| <= ||x_t|| ||w_e|| (Cauchy-Schwarz),
// four in-order fp32 chains of d/4 terms and three adds err by at most
// (d/4 + 3) 2^-24 P; a tcgen05 kind::f16 instruction adds 16 exact products
// to the fp32 accumulator losing at most one unit in the 2^-23 place of the
// largest of its 17 addends for each addend, plus one rounding of the sum,
// i.e. at most 18 2^-23 P per instruction over d/16 instructions; the total
// 1.25 d 2^-23 P is rounded up to 2 d 2^-23 P, and the norms (fp32 sums of
// exact squares) are enlarged by d 2^-23 before the square root.
//
// If |v_a - v_b| > 2 B_t, the order of a and b is the same under v and
// under f. So the refinement writes f over v for every expert whose order
// against another "candidate" of the token is not decided by v, where the
// candidates are the experts with v >= (k-th largest v) - 2 B_t: every other
// expert lies below each of the k experts that v ranks highest under both v
// and f. Every comparison the top-k makes between the mixed values then
// agrees with the one it makes on f (ties included, which can only occur
// between two rewritten values), so idx, the order of j and therefore all
// routing metadata equal those of the fixed-order logits. Gates are taken
// from the mixed values. A token whose bound is not finite (an inf or NaN in
// x or Wr) has all of its logits rewritten.
//
// One CTA handles RF_TOK tokens.
// Phase 1: a group of G lanes per token (32/G tokens per warp at a time),
// each lane holding the logits of experts g, g + G, ... in registers: k + 1
// rounds of a group maximum give the k + 1 largest v in descending order;
// listed are the winners among the first k whose neighbour in that order
// lies within 2 B_t, and every other expert within 2 B_t below the k-th.
// Phase 2: the tokens, ordered by the length of their lists so that a
// warp's tokens carry similar counts, go to 8 threads each: (quarter q,
// half h), the thread running the fmaf chains of quarter q for the listed
// experts h, h + 2, ... (up to RF_NPT at once, in registers, sharing its x
// values). The weight columns of each step (all experts, 4 quarters, RF_CK
// columns) are staged in shared memory by coalesced cp.async, double
// buffered; the four quarter sums of an expert meet by shuffles and are
// added ((c0 + c1) + c2) + c3.
constexpr int RF_TOK = 32;
constexpr int RF_THREADS = 256;  // 8 per token in phase 2
constexpr int RF_NPT = 8;        // listed experts per thread per pass (16 per token)

__host__ __device__ constexpr int rf_group_of(int E) {
    return E <= 8 ? 1 : E <= 16 ? 2 : E <= 32 ? 4 : E <= 64 ? 8 : E <= 128 ? 16 : 32;
}
// columns of each quarter staged per step, and the pitch of a staged row
__host__ __device__ constexpr int rf_ck(int E) { return E <= 64 ? 32 : E <= 128 ? 16 : 8; }
__host__ __device__ constexpr int rf_pitch(int E) { return 2 * rf_ck(E) + 16; }
inline size_t rf_smem_bytes(int64_t E) {
    return 2 * (size_t)E * 4 * (size_t)rf_pitch((int)E)       // phase 2 stages
           + sizeof(int16_t) * (size_t)RF_TOK * (size_t)E;  // per-token lists
}

__device__ __forceinline__ float rf_key(float a) { return a == a ? a : -INFINITY; }

// 8 bf16 (a 16-byte vector, element 0 in the low half of the first word)
// to fp32: one shift or mask per element, exact.
__device__ __forceinline__ void rf_unpack8(const uint4& u, float* f) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

// One staged step of NP chains (branch-free, so the chains interleave):
// acc[p] runs fmaf over x[j] * w_p[j] for the step's CK columns in
// ascending j; x comes from registers, w_p from the staged row at woff[p].
template <int NP, int CK>
__device__ __forceinline__ void rf_step(const uint4* xv, const unsigned char* wbase,
                                        const uint32_t* woff, float* acc) {
#pragma unroll
    for (int j8 = 0; j8 < CK / 8; ++j8) {
        float xf[8];
        rf_unpack8(xv[j8], xf);
        uint4 wv[NP];
#pragma unroll
        for (int p = 0; p < NP; ++p)
            wv[p] = *reinterpret_cast<const uint4*>(wbase + woff[p] + 16 * j8);
#pragma unroll
        for (int p = 0; p < NP; ++p) {
            float wf[8];
            rf_unpack8(wv[p], wf);
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[p] = fmaf(xf[j], wf[j], acc[p]);
        }
    }
}

template <int G>
__global__ void __launch_bounds__(RF_THREADS, 3) refine_kernel(
    const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ Wr,
    const float* __restrict__ xnorm2, const float* __restrict__ wnorm2, int T, int d, int E,
    int k, float* __restrict__ logits) {
    // logits per lane: rf_group_of gives G lanes to at most 8 G experts (16 G at G = 32)
    constexpr int VPL = G == 32 ? MOE_MAX_EXPERTS / 32 : 8;
    extern __shared__ __align__(16) unsigned char rf_smem[];
    unsigned char* s_w = rf_smem;  // [2][E][4][pitch]: phase 2 stages
    int16_t* s_list = reinterpret_cast<int16_t*>(
        rf_smem + 2 * (size_t)E * 4 * rf_pitch(E));  // [RF_TOK][E]: listed experts
    __shared__ int s_na[RF_TOK];
    __shared__ int s_order[RF_TOK];
    __shared__ int s_win_e[RF_TOK * (MOE_MAX_TOPK + 1)];
    __shared__ float s_win_v[RF_TOK * (MOE_MAX_TOPK + 1)];
    __shared__ int s_maxna;
    __shared__ float s_wmax;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int t0 = blockIdx.x * RF_TOK;

    if (warp == 0) {
        float m = 0.f;
        for (int e = lane; e < E; e += 32) {
            const float v = wnorm2[e];
            m = v == v ? fmaxf(m, v) : INFINITY;  // a NaN norm leaves no finite bound
        }
        m = warp_max(m);
        if (lane == 0) s_wmax = m;
    }
    if (tid < RF_TOK) s_na[tid] = 0;
    __syncthreads();
    const float infl = 1.f + (float)d * 0x1p-23f;
    const float wn = sqrtf(s_wmax * infl);

    // ---------------------------------------------------------- phase 1
    const int g = lane % G;
    for (int tl = tid / G; tl < RF_TOK; tl += RF_THREADS / G) {
        const int t = t0 + tl;
        int16_t* lst = s_list + (size_t)tl * E;
        const bool live = t < T;  // the same on every lane of the group
        float v[VPL];
#pragma unroll
        for (int i = 0; i < VPL; ++i) {
            const int e = g + G * i;
            v[i] = (live && e < E) ? rf_key(logits[(size_t)t * E + e]) : -INFINITY;
        }
        const float xn = live ? sqrtf(xnorm2[t] * infl) : 0.f;
        const float gap = 4.f * (float)d * 0x1p-23f * xn * wn * (1.f + 0x1p-20f);  // 2 B_t
        const bool all = live && !(gap <= 3.0e38f);  // no finite bound: every expert
        // k + 1 rounds of a group maximum (lower expert first on ties), each
        // retiring the winner: the k + 1 largest v in descending order
        int* win_e = s_win_e + tl * (MOE_MAX_TOPK + 1);
        float* win_v = s_win_v + tl * (MOE_MAX_TOPK + 1);
        uint32_t taken = 0, top = 0;  // top: this lane's experts among the first k
        const int rounds = k < E ? k + 1 : k;
        for (int r = 0; r < rounds; ++r) {
            if (r == k) top = taken;
            float bv = -INFINITY;
            int be = 0x7fffffff;
#pragma unroll
            for (int i = 0; i < VPL; ++i) {
                const int e = g + G * i;
                if (e < E && !((taken >> i) & 1u) && (be == 0x7fffffff || v[i] > bv)) {
                    bv = v[i];
                    be = e;
                }
            }
#pragma unroll
            for (int o = 1; o < G; o <<= 1) {
                const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
                const int oe = __shfl_xor_sync(0xffffffffu, be, o);
                if (ov > bv || (ov == bv && oe < be)) {
                    bv = ov;
                    be = oe;
                }
            }
            if (be < E && be % G == g) taken |= 1u << (be / G);
            if (g == 0) {
                win_e[r] = be;
                win_v[r] = bv;
            }
        }
        if (rounds == k) {  // k == E: nothing lies below the k-th
            top = taken;
            if (g == 0) win_v[k] = -INFINITY;
        }
        __syncwarp();
        // Listed: every expert when there is no finite bound; else each of the
        // k winners whose neighbour in the descending order lies within 2 B_t,
        // and every other expert within 2 B_t below the k-th winner (which
        // is then listed too). A difference of two nearby floats is exact,
        // so the tests below round nothing that could move an expert across
        // the 2 B_t line.
        if (live) {
            const float kth = win_v[k - 1];
            for (int r = g; r < k; r += G) {
                const float vr = win_v[r];
                const bool a = all || (r > 0 && win_v[r - 1] - vr <= gap) ||
                               (vr - win_v[r + 1] <= gap);
                if (a) lst[atomicAdd(&s_na[tl], 1)] = (int16_t)win_e[r];
            }
#pragma unroll
            for (int i = 0; i < VPL; ++i) {
                const int e = g + G * i;
                if (e < E && !((top >> i) & 1u) && (all || kth - v[i] <= gap))
                    lst[atomicAdd(&s_na[tl], 1)] = (int16_t)e;
            }
        }
        __syncwarp();
    }
    __syncthreads();
    if (tid < RF_TOK) {
        // rank by descending count (ties by token): s_order[rank] = token
        const int mine = s_na[tid];
        int rank = 0;
        for (int j = 0; j < RF_TOK; ++j) {
            const int o = s_na[j];
            rank += (o > mine) || (o == mine && j < tid);
        }
        s_order[rank] = tid;
        if (rank == 0) s_maxna = mine;
    }
    __syncthreads();

    // ---------------------------------------------------------- phase 2
    const int maxna = s_maxna;
    if (maxna == 0) return;
    const int tl = s_order[tid >> 3];
    const int q = (tid >> 1) & 3, h = tid & 1;
    const int t = t0 + tl;
    const int na = s_na[tl];
    const int dq = d >> 2;
    constexpr int CK = G <= 8 ? 32 : G == 16 ? 16 : 8;  // rf_ck(E) for the E this G serves
    const int pitch = rf_pitch(E);
    const int nsteps = dq / CK;
    const int chunks = E * 4 * (CK / 8);  // 16-byte pieces of one stage
    const uint32_t sw = smem_u32(s_w);
    const uint32_t stage_bytes = (uint32_t)E * 4u * (uint32_t)pitch;
    static_assert(RF_NPT == 8, "rf_step dispatch covers 1..8 chains");
    const uint4* xr = reinterpret_cast<const uint4*>(x + (size_t)(t < T ? t : 0) * d + (size_t)q * dq);
    auto stage = [&](int step, int buf) {
        const int c0 = step * CK;
        for (int i = tid; i < chunks; i += RF_THREADS) {
            const int row = i / (CK / 8), part = i - row * (CK / 8);  // row = 4 e + quarter
            const __nv_bfloat16* src =
                Wr + (size_t)(row >> 2) * d + (size_t)(row & 3) * dq + c0 + 8 * part;
            cp_async16(sw + buf * stage_bytes + row * pitch + 16 * part, src, 16);
        }
        cp_async_commit();
    };
    for (int pbase = 0; pbase < maxna; pbase += 2 * RF_NPT) {
        int cnt = 0;
        int ep[RF_NPT];
        uint32_t woff[RF_NPT];
#pragma unroll
        for (int p = 0; p < RF_NPT; ++p) {
            const int pi = pbase + 2 * p + h;
            ep[p] = pi < na ? (int)s_list[(size_t)tl * E + pi] : 0;
            woff[p] = (uint32_t)(ep[p] * 4 + q) * (uint32_t)pitch;  // expert 0 for unused slots
            if (pi < na) cnt = p + 1;
        }
        // chains per thread in this warp (the rest compute and drop expert 0's)
        const int npw = __reduce_max_sync(0xffffffffu, (unsigned)cnt);
        float acc[RF_NPT];
#pragma unroll
        for (int p = 0; p < RF_NPT; ++p) acc[p] = 0.f;
        __syncthreads();  // the previous pass is done with both stage buffers
        stage(0, 0);
        for (int st = 0; st < nsteps; ++st) {
            uint4 xv[CK / 8];
            if (npw > 0) {
#pragma unroll
                for (int u = 0; u < CK / 8; ++u) xv[u] = xr[(st * CK) / 8 + u];
            }
            if (st + 1 < nsteps) {
                stage(st + 1, (st + 1) & 1);
                cp_async_wait_one();
            } else {
                cp_async_wait_all();
            }
            __syncthreads();
            const unsigned char* wb = s_w + (st & 1) * stage_bytes;
            switch (npw) {
                case 0: break;
                case 1: rf_step<1, CK>(xv, wb, woff, acc); break;
                case 2: rf_step<2, CK>(xv, wb, woff, acc); break;
                case 3: rf_step<3, CK>(xv, wb, woff, acc); break;
                case 4: rf_step<4, CK>(xv, wb, woff, acc); break;
                case 5: rf_step<5, CK>(xv, wb, woff, acc); break;
                case 6: rf_step<6, CK>(xv, wb, woff, acc); break;
                case 7: rf_step<7, CK>(xv, wb, woff, acc); break;
                default: rf_step<8, CK>(xv, wb, woff, acc); break;
            }
            __syncthreads();  // before the next stage overwrites this buffer
        }
        // quarters q = 0..3 of (token, h) are lanes 8m + 2q + h
#pragma unroll
        for (int p = 0; p < RF_NPT; ++p) {
            const float c1 = __shfl_sync(0xffffffffu, acc[p], lane + 2);
            const float c2 = __shfl_sync(0xffffffffu, acc[p], lane + 4);
            const float c3 = __shfl_sync(0xffffffffu, acc[p], lane + 6);
            if (q == 0 && p < cnt && t < T) logits[(size_t)t * E + ep[p]] = ((acc[p] + c1) + c2) + c3;
        }
    }
}

template <int G>
static int launch_refine(const void* x, const void* Wr, const float* xnorm2, const float* wnorm2,
                         int64_t T, int64_t d, int64_t E, int k, float* logits, cudaStream_t st) {
    auto kern = refine_kernel<G>;
    static bool attr_done[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_done[dev]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)rf_smem_bytes(MOE_MAX_EXPERTS)) != cudaSuccess)
            return MOE_ERR_CUDA;
        attr_done[dev] = true;
    }
    const unsigned grid = (unsigned)((T + RF_TOK - 1) / RF_TOK);
    kern<<<grid, RF_THREADS, rf_smem_bytes(E), st>>>(
        static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(Wr), xnorm2,
        wnorm2, (int)T, (int)d, (int)E, k, logits);
    return MOE_OK;
}

static int launch_refine_any(const void* x, const void* Wr, const float* xnorm2,
                             const float* wnorm2, int64_t T, int64_t d, int64_t E, int k,
                             float* logits, cudaStream_t st) {
    switch (rf_group_of((int)E)) {
        case 1: return launch_refine<1>(x, Wr, xnorm2, wnorm2, T, d, E, k, logits, st);
        case 2: return launch_refine<2>(x, Wr, xnorm2, wnorm2, T, d, E, k, logits, st);
        case 4: return launch_refine<4>(x, Wr, xnorm2, wnorm2, T, d, E, k, logits, st);
        case 8: return launch_refine<8>(x, Wr, xnorm2, wnorm2, T, d, E, k, logits, st);
        case 16: return launch_refine<16>(x, Wr, xnorm2, wnorm2, T, d, E, k, logits, st);
        default: return launch_refine<32>(x, Wr, xnorm2, wnorm2, T, d, E, k, logits, st);
    }
}

// ------------------------------------------------------------------ a1

// Top-k on G lanes per token. Lane g of a token's group holds the logits of
// experts g*VPL .. g*VPL + VPL - 1 in registers (VPL a multiple of 8, at
// most 32). G starts at the smallest power of two with 32*G >= E and is
// doubled, while each lane keeps at least 8 logits and G <= 16, until the
// launch has about 1024 threads per SM: the selection is a chain of
// dependent steps, so it is latency-bound and wants many warps. A token's k
// selections are k rounds of: a tournament over the lane's untaken logits
// (lower expert first on equal values), then a butterfly over the G lanes of
// the group. The order is total (larger logit first, then lower index), so
// every lane of the group agrees on the winner and the result is the stable
// descending sort's first k. NaN stands for "taken or absent" inside the
// kernel; an input NaN is read as -inf (ranks below every number).
//
// One CTA is one chunk of CH tokens (CH = 32 for G <= 4, 16 for G = 8, 8 for
// G = 16). The rounds only record (expert, logit) in shared memory; then
// each lane takes the selections j = g, g + G, ...: it sets the token's bit
// in the shared-memory mask of the expert, computes the gate and writes idx
// and gate. After a barrier the rank of (t, e) within the chunk is the
// count of the mask's bits below t, and popc of the whole mask is the chunk
// count ws_count[e][chunk].
//
// The logits are read from NP planes pstride floats apart and added in
// plane order ((p0 + p1) + p2) + p3 (NP = 4: the router's quarter chains;
// 1: logits given by the caller); logits_out, when not null, receives the
// sums.
constexpr int TOPK_MAX_G = 16;
constexpr int topk_threads_of(int G) { return 32 * G < 128 ? 32 * G : 128; }

__device__ __forceinline__ bool is_num(float a) { return a == a; }

// (bv, be) <- the better of itself and (ov, oe); NaN never wins.
__device__ __forceinline__ void keep_better(float ov, int oe, float& bv, int& be) {
    const bool o_wins = is_num(ov) && (!is_num(bv) || ov > bv || (ov == bv && oe < be));
    bv = o_wins ? ov : bv;
    be = o_wins ? oe : be;
}

template <int G, int VPL, int NP>
__global__ void __launch_bounds__(topk_threads_of(G), 1) topk_group_kernel(
    const float* __restrict__ src, int64_t pstride, int vec, int T, int E, int k, int renorm,
    int nchunks, float* __restrict__ logits_out, int32_t* __restrict__ idx,
    float* __restrict__ gate, int32_t* __restrict__ rank, int32_t* __restrict__ ws_count) {
    constexpr int NT = topk_threads_of(G);
    constexpr int CH = NT / G;  // tokens per chunk (<= 32: one mask word per expert)
    __shared__ uint32_t hits[32 * G];
    __shared__ int32_t sel[CH][MOE_MAX_TOPK];  // selected expert of round j
    __shared__ float sval[CH][MOE_MAX_TOPK];   // its logit, then its gate
    const int c = blockIdx.x;
    const int g = threadIdx.x % G;
    const int tl = threadIdx.x / G;
    const int t = c * CH + tl;
    const bool live = t < T;
    for (int i = threadIdx.x; i < E; i += NT) hits[i] = 0u;

    const int e0 = g * VPL;
    float v[VPL];
#pragma unroll
    for (int q = 0; q < VPL; ++q) v[q] = __int_as_float(0x7fc00000);
    if (live) {
        const float* row = src + (size_t)t * E;
        if (vec) {
#pragma unroll
            for (int q = 0; q < VPL; q += 4) {
                if (e0 + q < E) {  // E % 4 == 0: the whole float4 is in the row
                    float4 a = __ldg(reinterpret_cast<const float4*>(row + e0 + q));
#pragma unroll
                    for (int p = 1; p < NP; ++p) {
                        const float4 b =
                            __ldg(reinterpret_cast<const float4*>(row + p * pstride + e0 + q));
                        a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w;
                    }
                    v[q] = a.x; v[q + 1] = a.y; v[q + 2] = a.z; v[q + 3] = a.w;
                    if (logits_out)
                        *reinterpret_cast<float4*>(logits_out + (size_t)t * E + e0 + q) = a;
                }
            }
        } else {
#pragma unroll
            for (int q = 0; q < VPL; ++q) {
                if (e0 + q < E) {
                    float a = __ldg(row + e0 + q);
#pragma unroll
                    for (int p = 1; p < NP; ++p) a += __ldg(row + p * pstride + e0 + q);
                    v[q] = a;
                    if (logits_out) logits_out[(size_t)t * E + e0 + q] = a;
                }
            }
        }
#pragma unroll
        for (int q = 0; q < VPL; ++q)
            if (e0 + q < E && !is_num(v[q])) v[q] = -INFINITY;
    }

    // softmax denominator: max over the group, then a pairwise sum of the
    // lane's exp terms and a butterfly over the group
    float mx = v[0];
#pragma unroll
    for (int q = 1; q < VPL; ++q) mx = fmaxf(mx, v[q]);
#pragma unroll
    for (int o = 1; o < G; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float s;
    {
        float ex[VPL];
#pragma unroll
        for (int q = 0; q < VPL; ++q) ex[q] = is_num(v[q]) ? expf(v[q] - mx) : 0.f;
#pragma unroll
        for (int w = 1; w < VPL; w <<= 1)
#pragma unroll
            for (int q = 0; q + w < VPL; q += 2 * w) ex[q] += ex[q + w];
        s = ex[0];
    }
#pragma unroll
    for (int o = 1; o < G; o <<= 1) s += __shfl_xor_sync(0xffffffffu, s, o);

    for (int j = 0; j < k; ++j) {
        // tournament over the lane's logits; on equal values the lower slot
        // (lower expert) is kept
        float tv[VPL];
        int tq[VPL];
#pragma unroll
        for (int q = 0; q < VPL; ++q) {
            tv[q] = v[q];
            tq[q] = q;
        }
#pragma unroll
        for (int w = 1; w < VPL; w <<= 1)
#pragma unroll
            for (int q = 0; q + w < VPL; q += 2 * w) {
                const bool r = is_num(tv[q + w]) && !(tv[q + w] <= tv[q]);
                tv[q] = r ? tv[q + w] : tv[q];
                tq[q] = r ? tq[q + w] : tq[q];
            }
        float bv = tv[0];
        int be = e0 + tq[0];
#pragma unroll
        for (int o = 1; o < G; o <<= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int oe = __shfl_xor_sync(0xffffffffu, be, o);
            keep_better(ov, oe, bv, be);
        }
        // the owner lane retires the winner; lane j % G records it
        const int qq = be - e0;
#pragma unroll
        for (int q = 0; q < VPL; ++q)
            if (q == qq) v[q] = __int_as_float(0x7fc00000);
        if (g == (j & (G - 1))) {
            sel[tl][j] = be;
            sval[tl][j] = bv;
        }
    }
    // each lane finishes its own selections j = g, g + G, ...; with renorm
    // the gates are written after the barrier, divided by their sum
    const uint32_t bit = 1u << tl;
    __syncthreads();  // every thread's share of the masks is zeroed
    if (live) {
        for (int j = g; j < k; j += G) {
            const int e = sel[tl][j];
            const float gj = expf(sval[tl][j] - mx) / s;
            sval[tl][j] = gj;
            atomicOr(&hits[e], bit);
            idx[(size_t)t * k + j] = e;
            if (!renorm) gate[(size_t)t * k + j] = gj;
        }
    }
    __syncthreads();
    if (live) {
        float gsum = 0.f;
        if (renorm)
            for (int j = 0; j < k; ++j) gsum += sval[tl][j];
        for (int j = g; j < k; j += G) {
            rank[(size_t)t * k + j] = __popc(hits[sel[tl][j]] & (bit - 1u));
            if (renorm) gate[(size_t)t * k + j] = sval[tl][j] / gsum;
        }
    }
    for (int e = threadIdx.x; e < E; e += NT) ws_count[(size_t)e * nchunks + c] = __popc(hits[e]);
}


// ------------------------------------------------------------------ a2

constexpr int SCAN_THREADS = 256;
constexpr int SCAN_ITEMS = 4;

// Block-wide exclusive scan of one int per thread (SCAN_THREADS threads).
__device__ int block_exclusive_scan(int v, int* total, int* sh /*[32]*/) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    int wt;
    int ex = warp_exclusive_scan(v, &wt);
    if (lane == 0) sh[w] = wt;
    __syncthreads();
    if (w == 0) {
        int x = lane < SCAN_THREADS / 32 ? sh[lane] : 0;
        int tt;
        int e2 = warp_exclusive_scan(x, &tt);
        if (lane < SCAN_THREADS / 32) sh[lane] = e2;
        if (lane == 0) sh[31] = tt;
    }
    __syncthreads();
    const int r = ex + sh[w];
    *total = sh[31];
    __syncthreads();
    return r;
}

__global__ void __launch_bounds__(SCAN_THREADS) scan_kernel(int E, int nchunks,
                                                            int32_t* __restrict__ ws_count,
                                                            int32_t* __restrict__ counts,
                                                            int32_t* __restrict__ offsets,
                                                            int32_t* __restrict__ tile_offsets,
                                                            int32_t* __restrict__ ticket) {
    __shared__ int sh[32];
    __shared__ int is_last;
    const int e = blockIdx.x;
    int32_t* row = ws_count + (size_t)e * nchunks;
    int carry = 0;
    for (int base = 0; base < nchunks; base += SCAN_THREADS * SCAN_ITEMS) {
        int v[SCAN_ITEMS];
        int local = 0;
        const int b0 = base + threadIdx.x * SCAN_ITEMS;
#pragma unroll
        for (int i = 0; i < SCAN_ITEMS; ++i) {
            v[i] = (b0 + i < nchunks) ? row[b0 + i] : 0;
            local += v[i];
        }
        int tot;
        int ex = block_exclusive_scan(local, &tot, sh) + carry;
#pragma unroll
        for (int i = 0; i < SCAN_ITEMS; ++i) {
            if (b0 + i < nchunks) row[b0 + i] = ex;
            ex += v[i];
        }
        carry += tot;
    }
    if (threadIdx.x == 0) {
        counts[e] = carry;
        __threadfence();
        const int prev = atomicAdd(ticket, 1);
        is_last = (prev == (int)gridDim.x - 1);
    }
    __syncthreads();
    if (!is_last) return;
    __threadfence();
    // last block: offsets and tile offsets over E <= 512 experts, 2 per thread
    int c0 = 0, c1 = 0;
    const int i0 = threadIdx.x * 2;
    if (i0 < E) c0 = __ldcg(counts + i0);
    if (i0 + 1 < E) c1 = __ldcg(counts + i0 + 1);
    int tot;
    int ex = block_exclusive_scan(c0 + c1, &tot, sh);
    if (i0 < E) offsets[i0] = ex;
    if (i0 + 1 < E) offsets[i0 + 1] = ex + c0;
    if (threadIdx.x == 0) offsets[E] = tot;
    if (tile_offsets) {
        const int m0 = (c0 + MOE_TILE_M - 1) / MOE_TILE_M, m1 = (c1 + MOE_TILE_M - 1) / MOE_TILE_M;
        int mt;
        int mex = block_exclusive_scan(m0 + m1, &mt, sh);
        if (i0 < E) tile_offsets[i0] = mex;
        if (i0 + 1 < E) tile_offsets[i0 + 1] = mex + m0;
        if (threadIdx.x == 0) tile_offsets[E] = mt;
    }
    if (threadIdx.x == 0) *ticket = 0;
}

__global__ void finalize_kernel(int T, int k, int E, int chunk, int nchunks,
                                const int32_t* __restrict__ idx,
                                const int32_t* __restrict__ offsets,
                                const int32_t* __restrict__ ws_count, int32_t* __restrict__ slot,
                                int* status) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t n = (int64_t)T * k;
    if (i >= n) return;
    const int t = (int)(i / k);
    const int e = idx[i];
    if (e < 0 || e >= E) {
        set_status(status, MOE_DEVERR_BAD_INDEX);
        return;
    }
    const int c = t / chunk;
    slot[i] = offsets[e] + ws_count[(size_t)e * nchunks + c] + slot[i];
}

// ------------------------------------------------------------------ host

// The chunk counts are sized for the smallest chunk (8 tokens, E > 256), so
// the workspace is a function of (T, E, from_x) alone.
constexpr int MIN_CHUNK = 8;
inline int64_t max_chunks_of(int64_t T) { return (T + MIN_CHUNK - 1) / MIN_CHUNK; }

inline size_t align256(size_t b) { return (b + 255) & ~size_t(255); }

struct RouteWs {
    int32_t* count;
    int32_t* ticket;
    float* planes;  // four [T,E] planes when the logits are computed
    float* xnorm2;  // [T] squared row norms of x (bf16 router)
    float* wnorm2;  // [E] squared row norms of Wr (bf16 router)
};

// from_x: the logits are computed from x and Wr; the workspace then also
// holds four [T,E] planes: the fp32 router's quarter chains (the top-k adds
// them), or in the first plane the bf16 router's logits when the caller does
// not ask for them.
inline int64_t plane_stride(int64_t T, int64_t E) { return (T * E + 63) / 64 * 64; }

inline size_t workspace_bytes(int64_t T, int64_t E, bool from_x) {
    size_t b = align256(sizeof(int32_t) * (size_t)E * (size_t)max_chunks_of(T));
    b += 256;  // ticket
    if (from_x) {
        b += align256(sizeof(float) * (size_t)LOGIT_SPLIT * (size_t)plane_stride(T, E));
        b += align256(sizeof(float) * (size_t)T) + align256(sizeof(float) * (size_t)E);
    }
    return b;
}

inline RouteWs carve(void* ws, int64_t T, int64_t E, bool from_x) {
    char* p = static_cast<char*>(ws);
    RouteWs r;
    r.count = reinterpret_cast<int32_t*>(p);
    p += align256(sizeof(int32_t) * (size_t)E * (size_t)max_chunks_of(T));
    r.ticket = reinterpret_cast<int32_t*>(p);
    p += 256;
    r.planes = nullptr;
    r.xnorm2 = r.wnorm2 = nullptr;
    if (from_x) {
        r.planes = reinterpret_cast<float*>(p);
        p += align256(sizeof(float) * (size_t)LOGIT_SPLIT * (size_t)plane_stride(T, E));
        r.xnorm2 = reinterpret_cast<float*>(p);
        p += align256(sizeof(float) * (size_t)T);
        r.wnorm2 = reinterpret_cast<float*>(p);
    }
    return r;
}

// Shape of the top-k launch for (T, E): lanes per token G, logits per lane
// V and tokens per chunk; chunk = 0 if no instantiation serves E.
struct TopkCfg {
    int G, V, chunk;
};
static TopkCfg topk_config(int64_t T, int64_t E) {
    TopkCfg c{1, 0, 0};
    if (E < 1 || E > MOE_MAX_EXPERTS) return c;
    while (32 * c.G < E) c.G *= 2;
    const int64_t want_threads = (int64_t)num_sms() * 1024;
    while (c.G < TOPK_MAX_G && T * c.G < want_threads && E >= 16 * c.G) c.G *= 2;
    c.V = (int)(((E + c.G - 1) / c.G + 7) / 8 * 8);
    if (c.G > TOPK_MAX_G || c.V < 8 || c.V > 32) return c;
    c.chunk = topk_threads_of(c.G) / c.G;
    return c;
}

// Launches the top-k with the shape topk_config chose; returns the chunk
// size (tokens per chunk).
static int launch_topk(const TopkCfg& cfg, const float* src, int nplanes, int64_t pstride, int T,
                       int E, int k, int renorm, float* logits_out, int32_t* idx, float* gate,
                       int32_t* rank, int32_t* wsc, cudaStream_t st) {
    const int G = cfg.G, V = cfg.V;
    const int nt = topk_threads_of(G);
    const int ch = nt / G;
    const int nch = (T + ch - 1) / ch;
    const int vec = (E % 4 == 0) && aligned16(src) && (!logits_out || aligned16(logits_out));
#define MOE_TOPK_NP(g, v, np)                                                                  \
    topk_group_kernel<g, v, np><<<nch, nt, 0, st>>>(src, pstride, vec, T, E, k, renorm, nch,  \
                                                    logits_out, idx, gate, rank, wsc)
#define MOE_TOPK_CASE(g, v)                                                                    \
    if (G == g && V == v) {                                                                    \
        if (nplanes == 4)                                                                      \
            MOE_TOPK_NP(g, v, 4);                                                              \
        else                                                                                   \
            MOE_TOPK_NP(g, v, 1);                                                              \
        return ch;                                                                             \
    }
#define MOE_TOPK_G(g) MOE_TOPK_CASE(g, 8) MOE_TOPK_CASE(g, 16) MOE_TOPK_CASE(g, 24) MOE_TOPK_CASE(g, 32)
    MOE_TOPK_G(1) MOE_TOPK_G(2) MOE_TOPK_G(4) MOE_TOPK_G(8) MOE_TOPK_G(16)
#undef MOE_TOPK_G
#undef MOE_TOPK_CASE
#undef MOE_TOPK_NP
    return 0;
}

}  // namespace route
}  // namespace moe

using namespace moe;

extern "C" size_t moe_route_workspace_size(int64_t T, int64_t E, int logits_from_x) {
    if (T < 0 || E <= 0) return 0;
    return route::workspace_bytes(T, E, logits_from_x != 0);
}

extern "C" int moe_route(const float* logits, const void* x, const void* Wr, int dtype, int64_t T,
                         int64_t d, int64_t E, int k, int renorm, float* logits_out, int32_t* idx,
                         float* gate, int32_t* counts, int32_t* offsets, int32_t* slot,
                         int32_t* tile_offsets, void* workspace, size_t workspace_bytes,
                         void* stream) {
    if (T < 0 || E < 1 || E > MOE_MAX_EXPERTS || k < 1 || k > MOE_MAX_TOPK || k > E)
        return MOE_ERR_INVALID;
    if (T * k > INT32_MAX || T > INT32_MAX / 2) return MOE_ERR_UNSUPPORTED;
    if (!counts || !offsets) return MOE_ERR_INVALID;
    if (T == 0) {
        // empty batch (an empty logits tensor may well be a null pointer): all
        // counts, offsets and tile offsets are zero
        if (check_only()) return MOE_OK;
        cudaStream_t st0 = as_stream(stream);
        if (cudaMemsetAsync(counts, 0, sizeof(int32_t) * E, st0) != cudaSuccess) return MOE_ERR_CUDA;
        if (cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (E + 1), st0) != cudaSuccess)
            return MOE_ERR_CUDA;
        if (tile_offsets &&
            cudaMemsetAsync(tile_offsets, 0, sizeof(int32_t) * (E + 1), st0) != cudaSuccess)
            return MOE_ERR_CUDA;
        return MOE_OK;
    }
    const bool from_x = (logits == nullptr);
    if (from_x) {
        if (!x || !Wr || d <= 0 || (d % route::LOGIT_D_ALIGN) != 0)
            return MOE_ERR_INVALID;
        if (dtype != MOE_F32 && dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
        if (!aligned16(x) || !aligned16(Wr)) return MOE_ERR_INVALID;
        if (d > (1 << 24)) return MOE_ERR_UNSUPPORTED;
    }
    if (T > 0 && (!idx || !gate || !slot)) return MOE_ERR_INVALID;
    if (!workspace || workspace_bytes < route::workspace_bytes(T, E, from_x))
        return MOE_ERR_INVALID;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MOE_ERR_INVALID;
    if (from_x && logits_out && (reinterpret_cast<uintptr_t>(logits_out) & 15u) != 0)
        return MOE_ERR_INVALID;
    const route::TopkCfg tk = route::topk_config(T, E);
    if (tk.chunk == 0) return MOE_ERR_UNSUPPORTED;
    if (check_only()) return MOE_OK;
    cudaStream_t st = as_stream(stream);
    route::RouteWs ws = route::carve(workspace, T, E, from_x);

    if (from_x && dtype == MOE_BF16) {
        // tensor cores, fp32 accumulation, with the row norms of x and Wr;
        // then the fixed-order logits of the experts whose order the tensor
        // core sums cannot decide; the top-k reads the one plane
        float* dst = logits_out ? logits_out : ws.planes;
        int rc = MOE_OK;
        if (E <= 64)
            rc = route::launch_router_tc<64>(x, Wr, T, d, E, dst, ws.xnorm2, ws.wnorm2, st);
        else if (E <= 128)
            rc = route::launch_router_tc<128>(x, Wr, T, d, E, dst, ws.xnorm2, ws.wnorm2, st);
        else
            rc = route::launch_router_tc<256>(x, Wr, T, d, E, dst, ws.xnorm2, ws.wnorm2, st);
        if (rc != MOE_OK) return rc;
        rc = route::launch_refine_any(x, Wr, ws.xnorm2, ws.wnorm2, T, d, E, k, dst, st);
        if (rc != MOE_OK) return rc;
        route::launch_topk(tk, dst, 1, 0, (int)T, (int)E, k, renorm, nullptr, idx, gate, slot,
                           ws.count, st);
    } else if (from_x) {
        // fp32 router: four fixed-order fmaf chains per logit on the CUDA
        // cores (tf32 tensor cores would round the inputs); the top-k adds
        // the four quarter planes
        dim3 grid((unsigned)((T + route::LOGIT_TT - 1) / route::LOGIT_TT),
                  (unsigned)((E + route::LOGIT_TE - 1) / route::LOGIT_TE), route::LOGIT_SPLIT);
        route::router_logits_kernel<<<grid, route::LOGIT_THREADS, 0, st>>>(
            static_cast<const float*>(x), static_cast<const float*>(Wr), (int)T, (int)d, (int)E,
            ws.planes, route::plane_stride(T, E));
        route::launch_topk(tk, ws.planes, route::LOGIT_SPLIT, route::plane_stride(T, E), (int)T,
                           (int)E, k, renorm, logits_out, idx, gate, slot, ws.count, st);
    } else {
        route::launch_topk(tk, logits, 1, 0, (int)T, (int)E, k, renorm, nullptr, idx, gate, slot,
                           ws.count, st);
    }
    const int chunk = tk.chunk;
    const int nch = (int)((T + chunk - 1) / chunk);
    if (cudaMemsetAsync(ws.ticket, 0, sizeof(int32_t), st) != cudaSuccess) return MOE_ERR_CUDA;
    route::scan_kernel<<<(unsigned)E, route::SCAN_THREADS, 0, st>>>(
        (int)E, nch, ws.count, counts, offsets, tile_offsets, ws.ticket);
    const int64_t n = T * k;
    route::finalize_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(
        (int)T, k, (int)E, chunk, nch, idx, offsets, ws.count, slot, status_ptr());
    return launch_status();
}
