/*
 * dropless top-k Mixture-of-Experts expert layer for NVIDIA B200 (sm_100a).
 *
 * C ABI. Every pointer argument named as "device" is caller-owned device
 * memory; the library never allocates, frees or synchronises (except
 * moe_get_status, which reads the device status word). All work is enqueued
 * on the caller's stream, passed as a `void*` holding a cudaStream_t
 * (NULL = legacy default stream). So any sequence of calls other than
 * moe_get_status and the *_host entries can be captured into a CUDA graph
 * and replayed (the replay reads the buffers' current contents); make one
 * call of each entry on the device before capturing, since the first call
 * sets kernel attributes.
 *
 * Notation: T tokens, d hidden size, E experts, k experts per token, F expert
 * FFN width, R = T*k rows of the expert-sorted buffers.
 *
 * Sources (page title, section) for what each call computes:
 *   [HF]  "Transformers 中的 OLMoE：稀疏 MoE 语言模型架构解析与推理实践"
 *         (blog.gitcode.com), §2 router, §3 experts, OlmoeConfig table.
 *   [OF]  "olmoforge" README (git.onestrm.cn/huzjie/olmoforge), capability
 *         table and MXFP8 block-quantisation sketch.
 *   [NEWS] "专家池 8→128 只慢 5%：Ai2 开源万亿参数 MoE 训练框架 Olmo-core 3"
 *         (xxqk.cn), section "三招拆分、三项优化、一个精度开关".
 *   [REL] "OLMo-core 3 发布：主攻混合专家训练与导出校验" (wedoingai.com),
 *         section "主要功能".
 *
 * Error behaviour (all calls): arguments are validated on the host before
 * anything is enqueued. MOE_ERR_INVALID / MOE_ERR_UNSUPPORTED mean nothing was
 * launched. The whole-layer entries (moe_layer_*), which chain the
 * single-step entries, first run every step's host checks without
 * enqueuing anything (the *_host entries do so for every token slice), so
 * an invalid argument of any step, such as a weight pointer of the last
 * GEMM that is not 16-byte aligned, is reported before the first launch.
 * MOE_ERR_CUDA means a CUDA call or launch failed (the CUDA error is left for
 * cudaGetLastError); work enqueued before it stays enqueued. Faults found on
 * the device (a metadata value out of range, a pipeline wait that exceeded
 * its time limit) set bits in a per-process device status word instead of
 * trapping; the kernel that finds one skips the bad access and returns. Read
 * it with moe_get_status. T == 0 is a valid no-op.
 *
 * Per-device state: on its first use on a device the library looks up and
 * keeps the device status word's address, sets kernel attributes, creates
 * the host pipeline's events and (moe_route_noalloc) looks up its scratch
 * array's address. A cudaDeviceReset, or any other teardown of the device's
 * primary context, invalidates all of it: do not call the library on a
 * device after resetting it.
 */
#ifndef DROPLESS_TOP_MIXTURE_B200_MOE_H
#define DROPLESS_TOP_MIXTURE_B200_MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

/* return codes */
#define MOE_OK 0
#define MOE_ERR_INVALID (-1)     /* bad argument, nothing launched            */
#define MOE_ERR_UNSUPPORTED (-2) /* shape/dtype outside what the build serves */
#define MOE_ERR_CUDA (-3)        /* a CUDA call or launch failed              */

/* element types */
#define MOE_F32 0
#define MOE_BF16 1
#define MOE_E4M3 2

/* MXFP8 scale encodings */
#define MOE_SCALE_F32 0  /* fp32 scale = amax/448 (1.0 for an all-zero block)      */
#define MOE_SCALE_E8M0 1 /* that value rounded up to a power of two, stored as the
                            biased exponent byte (e + 127)                       */

/* device status bits (moe_get_status) */
#define MOE_DEVERR_TIMEOUT 1      /* a bounded pipeline wait gave up           */
#define MOE_DEVERR_BAD_OFFSETS 2  /* offsets not monotone / not ending at R    */
#define MOE_DEVERR_BAD_INDEX 4    /* an expert index or slot out of range      */

/* limits of this build */
#define MOE_MAX_EXPERTS 512
#define MOE_MAX_TOPK 32
#define MOE_TILE_M 128 /* rows per M-tile of the grouped GEMM and tile table */

/* ------------------------------------------------------------------------
 * moe_route — router logits (optional), fp32 softmax, top-k, and the
 * GPU-resident routing metadata.
 *
 * [HF §2]: softmax over the E expert logits in fp32, torch.topk, optional
 * norm_topk_prob renormalisation (off by default per the OlmoeConfig table);
 * the router is a bias-free (E, d) weight. [OF capability table; NEWS]: the
 * routing table stays on the device so the host never waits for it.
 *
 * Inputs (device):
 *   logits   [T,E] fp32 row-major, or NULL to compute logits = x·Wrᵀ from
 *   x        [T,d] and Wr [E,d] in `dtype` (MOE_F32 or MOE_BF16). The
 *            routing is that of the fixed-order logits: the logit of (t,e)
 *            is four fp32 accumulators, one per contiguous quarter of j,
 *            each starting from +0.0 and updated by fused multiply-add in
 *            ascending j, then added in order, ((c0 + c1) + c2) + c3.
 *            fp32 inputs: computed that way on the CUDA cores (tf32 tensor
 *            cores would round the inputs). bf16 inputs (the pages' router
 *            is a linear layer in the model dtype): the tensor cores sum the
 *            exact products into fp32 in their own order, which differs from
 *            the fixed-order value by at most B_t = 2 d 2^-23 |x_t| max_e
 *            |w_e|; every expert of a token whose order against another
 *            candidate (an expert within 2 B_t of the k-th largest or above)
 *            is closer than 2 B_t is recomputed in the fixed order, so idx,
 *            the order of j and all metadata are exactly those of the
 *            fixed-order logits (finite inputs; a token whose bound is not
 *            finite has all E logits recomputed). The logits written out
 *            are the fixed-order values for the recomputed experts and the
 *            tensor-core sums for the others; the gates are computed from
 *            them.
 *   renorm   0: gates are the softmax probabilities; 1: divided by their sum.
 * Outputs (device, caller-allocated):
 *   logits_out  [T,E] fp32, or NULL (used only when logits == NULL)
 *   idx      [T,k] int32: expert indices by descending logit, ties to the
 *            lower index (selection on the fp32 logits; NaN ranks as -inf)
 *   gate     [T,k] fp32: softmax probability of idx[t,j] (fp32 arithmetic)
 *   counts   [E]   int32 rows per expert
 *   offsets  [E+1] int32 exclusive prefix sum of counts; offsets[E] = R
 *   slot     [T,k] int32 row of (t,j) in the expert-sorted buffers: rows of
 *            expert e are offsets[e].., in ascending token order
 *   tile_offsets [E+1] int32 exclusive prefix sum of ceil(counts/128), or NULL
 * Workspace: `workspace_bytes` >= moe_route_workspace_size(T, E,
 *            logits == NULL); 256-byte aligned device memory (with logits
 *            computed it holds four [T,E] fp32 planes: the fp32 router's
 *            quarter sums, or the bf16 router's logits when logits_out is
 *            NULL, and the squared row norms of x and Wr). Its contents need
 *            not be initialised.
 * Limits: 1 <= k <= min(E, 32), E <= 512; when computing logits d % 128 == 0
 *            and logits_out (if given) 16-byte aligned.
 * ---------------------------------------------------------------------- */
MOE_API size_t moe_route_workspace_size(int64_t T, int64_t E, int logits_from_x);
MOE_API int moe_route(const float* logits, const void* x, const void* Wr, int dtype, int64_t T,
                      int64_t d, int64_t E, int k, int renorm, float* logits_out, int32_t* idx,
                      float* gate, int32_t* counts, int32_t* offsets, int32_t* slot,
                      int32_t* tile_offsets, void* workspace, size_t workspace_bytes,
                      void* stream);

/* ------------------------------------------------------------------------
 * moe_route_noalloc — moe_route without a caller workspace.
 *
 * No counterpart in the pages: this is an interface convenience of this
 * library. It is for callers that cannot allocate device memory (an enqueue
 * callback that is given only tensors and a stream, or a process whose memory
 * pool owns the device, where cudaMalloc would synchronise or fail). It
 * computes exactly what moe_route computes, with the same arguments minus
 * `workspace`/`workspace_bytes`; its scratch is a library-owned device array
 * of MOE_ROUTE_NOALLOC_SCRATCH_BYTES that every GPU loading the library
 * keeps reserved until the process exits.
 *   - Size limit: moe_route_workspace_size(T, E, logits == NULL) must not
 *     exceed MOE_ROUTE_NOALLOC_SCRATCH_BYTES, else MOE_ERR_UNSUPPORTED and
 *     nothing is launched. (E = 64 with logits computed from x fits up to
 *     T = 7,913 tokens; E = 128 with logits given up to T = 131,064; E = 384
 *     with logits given up to T = 43,688.)
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current and caches it; make
 *     that first call before any stream capture begins.
 *   - All calls share the one array and it keeps the previous call's
 *     contents; calls whose work can overlap on the GPU (different streams
 *     without ordering, or different host threads) race on it and must be
 *     serialised by the caller.
 *   - It calls no cudaMalloc/cudaFree and allocates nothing.
 * ---------------------------------------------------------------------- */
#define MOE_ROUTE_NOALLOC_SCRATCH_BYTES (8u << 20)
MOE_API int moe_route_noalloc(const float* logits, const void* x, const void* Wr, int dtype,
                              int64_t T, int64_t d, int64_t E, int k, int renorm,
                              float* logits_out, int32_t* idx, float* gate, int32_t* counts,
                              int32_t* offsets, int32_t* slot, int32_t* tile_offsets,
                              void* stream);

/* ------------------------------------------------------------------------
 * moe_dispatch — row-wise dispatch: Xe[slot[t,j], :] = x[t, :].
 *
 * [OF capability table, row-wise expert parallelism]: each (token, k) row is
 * written straight into its expert's contiguous input buffer; there is no
 * separate permute. With `gate` non-NULL each copy is scaled:
 * Xe[slot[t,j]] = round_dtype(fp32(gate[t,j]) * x[t]) (used to form the
 * upstream gradient of the backward pass).
 *   x [T,d], Xe [R,d] in `dtype` (MOE_F32 or MOE_BF16), rows contiguous,
 *   16-byte aligned, d*elem_size % 16 == 0. slot [T,k] from moe_route.
 * A slot outside [0,R) is skipped and sets MOE_DEVERR_BAD_INDEX.
 * ---------------------------------------------------------------------- */
MOE_API int moe_dispatch(const void* x, const int32_t* slot, const float* gate, int64_t T,
                         int64_t d, int k, int dtype, void* Xe, void* stream);
/* moe_dispatch_gate — the unscaled dispatch that also records each expert
 * row's gate, row_gate[slot[t,j]] = gate[t,j] (fp32 [R], device), for
 * moe_grouped_down_gated. gate [T,k] and row_gate must be non-NULL when
 * T > 0; otherwise as moe_dispatch. */
MOE_API int moe_dispatch_gate(const void* x, const int32_t* slot, const float* gate, int64_t T,
                              int64_t d, int k, int dtype, void* Xe, float* row_gate,
                              void* stream);

/* ------------------------------------------------------------------------
 * moe_row_token — the inverse of the slot map: row_token[slot[t,j]] = t,
 * i.e. the token whose copy expert row r holds.
 *
 * [OF capability table, row-wise expert parallelism, "免重排" (no separate
 * permutation)]: with row_token a GEMM can fetch its expert rows straight
 * from x (moe_grouped_gate_up_gather), so the dispatched copy Xe is never
 * materialised.
 *   slot [T,k] from moe_route; row_token [R = T*k] int32 output.
 * A slot outside [0,R) is skipped and sets MOE_DEVERR_BAD_INDEX.
 * ---------------------------------------------------------------------- */
MOE_API int moe_row_token(const int32_t* slot, int64_t T, int k, int32_t* row_token,
                          void* stream);

/* ------------------------------------------------------------------------
 * Grouped SwiGLU expert FFN over variable per-expert row counts.
 *
 * [HF §3]: per expert e, rows r in [offsets[e], offsets[e+1]):
 *   H[r]  = silu(Xe[r]·W1_eᵀ) * (Xe[r]·W3_eᵀ)        (moe_grouped_gate_up)
 *   Ye[r] = H[r]·W2_eᵀ                                (moe_grouped_down)
 * [OF; NEWS]: all experts' small matmuls run as one grouped kernel.
 * Tensor-core (tcgen05) products with fp32 accumulation; MOE_BF16 operands
 * use bf16 MMA, MOE_F32 operands use tf32 MMA. H and Ye are stored in the
 * same dtype.
 *   Xe  [R,d]                      row-major
 *   W1, W3  expert e at W + e*w13_expert_stride elements, each [F,d]
 *           row-major (d contiguous). Separate [E,F,d] tensors use stride
 *           F*d; the fused gate/up layout [E,2F,d] of [HF §3] uses W1 =
 *           base, W3 = base + F*d, stride 2*F*d.
 *   W2  expert e at W2 + e*w2_expert_stride elements, [d,F] row-major.
 *   offsets [E+1] from moe_route (validated on the device: monotone, ending
 *           at R; otherwise MOE_DEVERR_BAD_OFFSETS and nothing is written).
 *   H   [R,F] device output/workspace; Ye [R,d] device output.
 * Limits: d % 128 == 0, F % 128 == 0, E <= 512; every pointer 16-byte
 * aligned; strides multiples of 8 elements.
 * Two tile forms compute the same sums in the same order (bit-identical
 * results): row tiles (128 or, for the down GEMM of experts averaging 512+
 * rows, 256 expert rows x 256 weight rows) and token-column tiles (256
 * weight rows x up to 256 of one expert's tokens, in steps of 16), chosen
 * by shape: token columns when experts average 512 rows or more and the
 * weight layout allows their maps (gate/up: the expert stride a multiple of
 * 16*d and W3 - W1 a nonzero multiple of 16 bytes; down: the expert stride
 * a multiple of F and d % 256 == 0), row tiles otherwise.
 * ---------------------------------------------------------------------- */
MOE_API int moe_grouped_gate_up(const void* Xe, const void* W1, const void* W3,
                                int64_t w13_expert_stride, const int32_t* offsets, int64_t E,
                                int64_t R, int64_t d, int64_t F, int dtype, void* H,
                                void* stream);
MOE_API int moe_grouped_down(const void* H, const void* W2, int64_t w2_expert_stride,
                             const int32_t* offsets, int64_t E, int64_t R, int64_t d, int64_t F,
                             int dtype, void* Ye, void* stream);
/* moe_grouped_down with the routing weights in its epilogue ([OF]
 * capability table; "Transformers 中的 OLMoE" §3 multiplies each expert's
 * output by its top-k weight): Ye[r] = round_dtype(row_gate[r] *
 * fp32(H[r]·W2_eᵀ)), so the combine adds the k rows of a token with unit
 * gates (moe_combine with gate = NULL). row_gate [R] fp32 from
 * moe_dispatch_gate, non-NULL when R > 0; otherwise as moe_grouped_down. */
MOE_API int moe_grouped_down_gated(const void* H, const void* W2, int64_t w2_expert_stride,
                                   const int32_t* offsets, const float* row_gate, int64_t E,
                                   int64_t R, int64_t d, int64_t F, int dtype, void* Ye,
                                   void* stream);
MOE_API int moe_grouped_swiglu(const void* Xe, const void* W1, const void* W3, const void* W2,
                               int64_t w13_expert_stride, int64_t w2_expert_stride,
                               const int32_t* offsets, int64_t E, int64_t R, int64_t d,
                               int64_t F, int dtype, void* H, void* Ye, void* stream);
/* moe_grouped_gate_up with the dispatch folded in: expert row r is token
 * row_token[r] of x [T,d] (moe_row_token), fetched by TMA row gathers
 * (tile::gather4, four 128-byte row pieces per copy) into the GEMM's A
 * tiles, so Xe is never written. H equals moe_grouped_gate_up on
 * moe_dispatch's Xe bit for bit. A row_token outside [0,T) is read as
 * token 0 and sets MOE_DEVERR_BAD_INDEX. Limits as moe_grouped_gate_up;
 * T >= 1 when R > 0. On B200 this is about 3x slower than moe_dispatch +
 * moe_grouped_gate_up (the row gathers, not the bytes, limit it), so
 * moe_layer_fwd does not use it. */
MOE_API int moe_grouped_gate_up_gather(const void* x, const int32_t* row_token, int64_t T,
                                       const void* W1, const void* W3,
                                       int64_t w13_expert_stride, const int32_t* offsets,
                                       int64_t E, int64_t R, int64_t d, int64_t F, int dtype,
                                       void* H, void* stream);
/* moe_grouped_gate_up with the pre-activations kept for the backward pass:
 * A_out[r] = Xe[r]·W1_eᵀ and B_out[r] = Xe[r]·W3_eᵀ ([R,F], layer dtype),
 * written by the same epilogue that writes H. Both NULL = moe_grouped_gate_up. */
MOE_API int moe_grouped_gate_up_save(const void* Xe, const void* W1, const void* W3,
                                     int64_t w13_expert_stride, const int32_t* offsets, int64_t E,
                                     int64_t R, int64_t d, int64_t F, int dtype, void* H,
                                     void* A_out, void* B_out, void* stream);

/* ------------------------------------------------------------------------
 * moe_grouped_swiglu_bwd — backward of the grouped SwiGLU FFN.
 *
 * ["OLMo-core 3 发布：主攻混合专家训练与导出校验", 主要功能: pairwise SwiGLU
 * backward and bf16 weight gradients.] Given the forward's saved rows Xe,
 * A = Xe·W1ᵀ, B = Xe·W3ᵀ, H = silu(A)*B and the upstream rows dYe [R,d]
 * (moe_dispatch of dOut with the gates), per expert e and its rows:
 *   dH  = dYe·W2_e;  dA = dH*B*silu'(A);  dB = dH*silu(A)   (silu'(a) =
 *         s(1 + a(1-s)), s = sigmoid(a); fused into the dH GEMM epilogue)
 *   dXe = dA·W1_e + dB·W3_e
 *   dW1_e = dAᵀ·Xe_e,  dW3_e = dBᵀ·Xe_e,  dW2_e = dYeᵀ·H_e
 * tcgen05 bf16 MMA, fp32 accumulation, every output stored in bf16.
 *   dA, dB [R,F] (outputs, also used as workspace), dXe [R,d];
 *   dW1, dW3 [E,F,d] and dW2 [E,d,F], contiguous; an expert with no rows
 *   gets zero gradients. Weights as in moe_grouped_gate_up/down.
 * Limits: MOE_BF16 only; d % 256 == 0, F % 256 == 0, E <= 512. Router and
 * gate gradients are not computed here.
 * ---------------------------------------------------------------------- */
MOE_API int moe_grouped_swiglu_bwd(const void* Xe, const void* A, const void* B, const void* H,
                                   const void* dYe, const void* W1, const void* W3,
                                   const void* W2, int64_t w13_expert_stride,
                                   int64_t w2_expert_stride, const int32_t* offsets, int64_t E,
                                   int64_t R, int64_t d, int64_t F, int dtype, void* dA, void* dB,
                                   void* dXe, void* dW1, void* dW3, void* dW2, void* stream);

/* moe_grouped_swiglu_wgrad: the weight-gradient GEMMs of
 * moe_grouped_swiglu_bwd alone (dW1_e = dAᵀ·Xe_e, dW3_e = dBᵀ·Xe_e,
 * dW2_e = dYeᵀ·H_e over each expert's rows; zeros for an expert with no
 * rows), from bf16 rows Xe, dYe [R,d] and dA, dB, H [R,F]. Same layouts and
 * limits as moe_grouped_swiglu_bwd. The MXFP8 backward runs it on the
 * forward's dequantised Xe and H. */
MOE_API int moe_grouped_swiglu_wgrad(const void* Xe, const void* dA, const void* dB,
                                     const void* dYe, const void* H, const int32_t* offsets,
                                     int64_t E, int64_t R, int64_t d, int64_t F, int dtype,
                                     void* dW1, void* dW3, void* dW2, void* stream);

/* ------------------------------------------------------------------------
 * moe_combine — gate-weighted combine back to token order.
 *
 * [HF §3]: each expert output is multiplied by its top-k weight and added
 * back at its token (index_add_). Here, per token, a gather:
 *   out[t] = round_dtype( sum_{j=0..k-1} gate[t,j] * Ye[slot[t,j]] )
 * accumulated in fp32 by fused multiply-add in ascending j, starting from 0.
 * gate == NULL means unit gates (used for the input gradient in backward).
 * No atomics: the result is deterministic.
 *   Ye [R,d], out [T,d] in `dtype`; rows 16-byte aligned.
 * ---------------------------------------------------------------------- */
MOE_API int moe_combine(const void* Ye, const int32_t* slot, const float* gate, int64_t T,
                        int64_t d, int k, int dtype, void* out, void* stream);

/* ------------------------------------------------------------------------
 * MXFP8 block quantisation [OF "MXFP8 分块量化"; NEWS].
 *
 * Blocks of 32 consecutive elements of each row share one scale:
 *   s = fp32(amax/448) (1.0 if amax == 0); MOE_SCALE_E8M0 rounds s up to
 *   the next power of two (exponent clamped to [-127,127]) and stores the
 *   byte e+127. Codes: q = E4M3(fp32(v/s)), round-to-nearest-even,
 *   saturating to ±448.
 *   in [rows, cols] MOE_F32 or MOE_BF16; cols % 32 == 0
 *   q [rows, cols] uint8 E4M3 codes; scales [rows, cols/32] fp32
 *   (MOE_SCALE_F32) or uint8 (MOE_SCALE_E8M0).
 * Dequantise: out_bf16 = bf16_rne(fp32(decode(q) * s)).
 * ---------------------------------------------------------------------- */
MOE_API int mxfp8_quantize(const void* in, int dtype, int64_t rows, int64_t cols,
                           int scale_mode, uint8_t* q, void* scales, void* stream);
MOE_API int mxfp8_dequantize(const uint8_t* q, const void* scales, int scale_mode,
                             int64_t rows, int64_t cols, void* out_bf16, void* stream);

/* ------------------------------------------------------------------------
 * MXFP8 path ["olmoforge" README, capability table and "MXFP8 分块量化";
 * "专家池 8→128 只慢 5%…", "三招拆分、三项优化、一个精度开关"].
 *
 * moe_dispatch_mxfp8: quantise each token row of x [T,d] (bf16) once, in
 *   blocks of 32 along d with UE8M0 scales (as mxfp8_quantize with
 *   MOE_SCALE_E8M0), and write codes and scales to its k slots:
 *   Xq [R,d] uint8 E4M3, Xs [R,d/32] uint8. d % 32 == 0.
 * moe_grouped_gate_up_mxfp8 / moe_grouped_down_mxfp8: the grouped SwiGLU
 *   FFN on block-scaled FP8 MMA (tcgen05 kind::mxf8f6f4, fp32 accumulate).
 *   Weights are E4M3 codes with UE8M0 scales along their contraction
 *   dimension (mxfp8_quantize of W1/W3 as [E*F, d] and W2 as [E*d, F]):
 *   W1q/W3q [E,F,d] + W1s/W3s [E,F,d/32]; W2q [E,d,F] + W2s [E,d,F/32];
 *   expert strides in elements of the code tensors. The GEMMs take the
 *   weight scales packed once by mxfp8_pack_weight_scales (below).
 *   The activation scales they read (Xs for gate/up, Hs for down) are in the
 *   tile-packed layout of mxfp8_pack_act_scales (below); gate/up writes H
 *   quantised from its fp32 value: Hq [R,F] codes and its scales Hs in that
 *   same tile-packed layout (K = F), ready for down; down writes Ye [R,d]
 *   bf16. Limits: d % 128 == 0, F % 128 == 0; code and scale pointers
 *   16-byte aligned.
 *
 * mxfp8_pack_weight_scales: the weight scales in the order the GEMMs'
 *   tensor-core scale copy reads them, so each pipeline stage fetches them
 *   with one bulk copy. For every expert, every 256-row B tile (gate/up:
 *   rows 128nb..128nb+127 of W1 then the same rows of W3; down: rows
 *   256nb..256nb+255 of W2, rows past d zero) and every 128-element K slab
 *   s, two 512-byte blocks (tile rows 0..127, then 128..255) each hold the
 *   four scale bytes (K blocks 4s..4s+3) of their row m at byte
 *   16*(m % 32) + 4*(m / 32); blocks ordered (expert, n-block, slab, half).
 *   Ps13: E*(F/128)*(d/128)*1024 bytes (from W1s, W3s); Ps2:
 *   E*ceil(d/256)*(F/128)*1024 bytes (from W2s). Either pair may be NULL.
 *   Scale tensors contiguous as above; packed outputs 16-byte aligned.
 *
 * mxfp8_pack_act_scales / mxfp8_unpack_act_scales: activation scales between
 *   the row layout S [R, K/32] (K-block bytes of each expert-sorted row, as
 *   moe_dispatch_mxfp8 and mxfp8_quantize write them) and the tile-packed
 *   layout Sp the GEMMs copy with one bulk copy per stage. The rows of
 *   expert e (offsets[e]..offsets[e+1], device int32 [E+1]) form
 *   ceil(count/128) row tiles, numbered over the experts in order; for row
 *   tile g and 128-element K slab s, the 512-byte block at (g*(K/128) + s)*512
 *   holds the word (four K-block bytes) of tile row m at 16*(m % 32) +
 *   4*(m / 32); tile rows past the expert's rows hold 0 (pack writes them;
 *   unpack ignores them). Sp takes mxfp8_act_scales_packed_size(E, R, K) =
 *   (R/128 + E)*(K/128)*512 bytes (an upper bound on the tiles; blocks past
 *   the last tile are not touched). K % 128 == 0; S and Sp 16-byte aligned;
 *   offsets not monotone from 0 to R set MOE_DEVERR_BAD_OFFSETS and nothing
 *   is written.
 * ---------------------------------------------------------------------- */
MOE_API int moe_dispatch_mxfp8(const void* x, const int32_t* slot, int64_t T, int64_t d, int k,
                               uint8_t* Xq, uint8_t* Xs, void* stream);
MOE_API int mxfp8_pack_weight_scales(const uint8_t* W1s, const uint8_t* W3s, const uint8_t* W2s,
                                     int64_t E, int64_t d, int64_t F, uint8_t* Ps13,
                                     uint8_t* Ps2, void* stream);
MOE_API size_t mxfp8_act_scales_packed_size(int64_t E, int64_t R, int64_t K);
MOE_API int mxfp8_pack_act_scales(const uint8_t* S, const int32_t* offsets, int64_t E, int64_t R,
                                  int64_t K, uint8_t* Sp, void* stream);
MOE_API int mxfp8_unpack_act_scales(const uint8_t* Sp, const int32_t* offsets, int64_t E,
                                    int64_t R, int64_t K, uint8_t* S, void* stream);
MOE_API int moe_grouped_gate_up_mxfp8(const uint8_t* Xq, const uint8_t* Xs, const uint8_t* W1q,
                                      const uint8_t* W3q, const uint8_t* Ps13,
                                      int64_t w13_expert_stride, const int32_t* offsets, int64_t E,
                                      int64_t R, int64_t d, int64_t F, uint8_t* Hq, uint8_t* Hs,
                                      void* stream);
MOE_API int moe_grouped_down_mxfp8(const uint8_t* Hq, const uint8_t* Hs, const uint8_t* W2q,
                                   const uint8_t* Ps2, int64_t w2_expert_stride,
                                   const int32_t* offsets, int64_t E, int64_t R, int64_t d,
                                   int64_t F, void* Ye, void* stream);
/* moe_grouped_gate_up_mxfp8_save: moe_grouped_gate_up_mxfp8 that also
 * stores the pre-activations A = Xe·W1ᵀ and B = Xe·W3ᵀ (the fp32
 * accumulators rounded to bf16, [R,F] each, 16-byte aligned) for the
 * backward; A_out and B_out both NULL is the plain call. */
MOE_API int moe_grouped_gate_up_mxfp8_save(const uint8_t* Xq, const uint8_t* Xs,
                                           const uint8_t* W1q, const uint8_t* W3q,
                                           const uint8_t* Ps13, int64_t w13_expert_stride,
                                           const int32_t* offsets, int64_t E, int64_t R,
                                           int64_t d, int64_t F, uint8_t* Hq, uint8_t* Hs,
                                           void* A_out, void* B_out, void* stream);

/* moe_layer_fwd_mxfp8 — route -> moe_dispatch_mxfp8 -> gate/up (MXFP8) ->
 * down (MXFP8) -> moe_combine (bf16), on one stream. x, Wr and out are bf16. */
typedef struct moe_layer_mxfp8_args {
    int64_t T, d, E, F;
    int32_t k, renorm, reserved0, reserved1;
    const void* x;          /* [T,d] bf16                                     */
    const float* logits;    /* [T,E] fp32, or NULL to use Wr                  */
    const void* Wr;         /* [E,d] bf16                                     */
    const uint8_t* W1q;
    const uint8_t* W3q;
    const uint8_t* W2q;
    const uint8_t* Ps13;    /* packed gate/up weight scales (mxfp8_pack_weight_scales) */
    const uint8_t* Ps2;     /* packed down weight scales                      */
    int64_t w13_expert_stride, w2_expert_stride;
    void* out;              /* [T,d] bf16                                     */
    int32_t* idx;
    float* gate;
    int32_t* counts;
    int32_t* offsets;
    int32_t* slot;
    void* workspace;        /* Xq, Xs (rows and tile-packed), Hq, Hs (packed),
                               Ye and the route workspace                     */
    size_t workspace_bytes;
    /* optional, all NULL or all set: the forward keeps what
     * moe_layer_bwd_mxfp8 needs in these caller buffers instead of the
     * workspace (R = T*k): Xq [R,d] codes, Xs [R,d/32] row-layout scales,
     * Hq [R,F] codes, Hsp tile-packed H scales
     * (mxfp8_act_scales_packed_size(E,R,F) bytes), A and B [R,F] bf16
     * pre-activations. Not accepted by moe_layer_fwd_mxfp8_host. */
    uint8_t* save_Xq;
    uint8_t* save_Xs;
    uint8_t* save_Hq;
    uint8_t* save_Hsp;
    void* save_A;
    void* save_B;
} moe_layer_mxfp8_args;

MOE_API size_t moe_layer_mxfp8_workspace_size(int64_t T, int64_t d, int64_t E, int64_t F, int k,
                                              int logits_given);
MOE_API int moe_layer_fwd_mxfp8(const moe_layer_mxfp8_args* args, void* stream);
/* moe_layer_fwd_mxfp8_host — moe_layer_fwd_mxfp8 from and to host memory in
 * token slices with the copies overlapped, exactly as moe_layer_fwd_host
 * (x and out are bf16 [T,d] host buffers; args->x, ->logits, ->out are the
 * device staging buffers). Every token's output equals the one-shot call's
 * bit for bit. */
MOE_API int moe_layer_fwd_mxfp8_host(const moe_layer_mxfp8_args* args, const void* x_host,
                                     const float* logits_host, void* out_host, int chunks,
                                     void* stream, void* stream_h2d, void* stream_d2h);

/* ------------------------------------------------------------------------
 * moe_layer_fwd — the whole layer: route -> dispatch -> grouped SwiGLU ->
 * combine [HF §2-§3], enqueued on one stream with no host synchronisation.
 * ---------------------------------------------------------------------- */
typedef struct moe_layer_args {
    int64_t T, d, E, F;
    int32_t k, dtype, renorm, reserved0;
    /* inputs (device) */
    const void* x;          /* [T,d]                                          */
    const float* logits;    /* [T,E] fp32, or NULL to use Wr                  */
    const void* Wr;         /* [E,d] (when logits == NULL)                    */
    const void* W1;         /* see moe_grouped_gate_up                        */
    const void* W3;
    const void* W2;
    int64_t w13_expert_stride, w2_expert_stride;
    /* outputs (device) */
    void* out;              /* [T,d]                                          */
    int32_t* idx;           /* [T,k]                                          */
    float* gate;            /* [T,k]                                          */
    int32_t* counts;        /* [E]                                            */
    int32_t* offsets;       /* [E+1]                                          */
    int32_t* slot;          /* [T,k]                                          */
    /* scratch (device): Xe [R,d], H [R,F], Ye [R,d], the rows' gates [R] and
     * the route workspace. Without save_Ye the layer applies the gates in
     * the down GEMM's epilogue (moe_dispatch_gate, moe_grouped_down_gated,
     * unit-gate combine); with save_Ye it keeps Ye unscaled for the router
     * backward and the combine applies the gates. */
    void* workspace;
    size_t workspace_bytes;
    /* optional (device, NULL = not kept): rows kept for moe_layer_bwd. When
     * save_Xe / save_H are given they replace the workspace copies; save_A and
     * save_B (given together) receive the gate/up pre-activations. */
    void* save_Xe;          /* [R,d] */
    void* save_H;           /* [R,F] */
    void* save_A;           /* [R,F] */
    void* save_B;           /* [R,F] */
    /* optional, for the router backward of moe_layer_bwd: the expert output
     * rows Ye [R,d] (replacing the workspace copy) and, when the logits are
     * computed from x and Wr, the fp32 logits [T,E] */
    void* save_Ye;
    float* save_logits;
} moe_layer_args;

MOE_API size_t moe_layer_workspace_size(int64_t T, int64_t d, int64_t E, int64_t F, int k,
                                        int dtype, int logits_given);
MOE_API int moe_layer_fwd(const moe_layer_args* args, void* stream);

/* ------------------------------------------------------------------------
 * moe_layer_fwd_host — moe_layer_fwd from and to host memory, with the
 * copies overlapped with compute. The layer is token-wise, so the batch is
 * cut into `chunks` consecutive token slices (<= 64): slice c is copied in
 * on `stream_h2d`, computed on `stream`, and copied out on `stream_d2h`, so
 * the copy-in of slice c+1 and the copy-out of slice c-1 run while slice c
 * computes. With three or more slices the first and the last hold half as
 * many tokens as the others (slice i ends at token T*(2i+1)/(2(chunks-1)),
 * the last at T), which shortens the copies nothing overlaps. Every token's
 * output equals moe_layer_fwd's bit for bit.
 *   args        as for moe_layer_fwd; args->x (and args->logits) and
 *               args->out are device staging buffers for the whole batch
 *               ([T,d], [T,E], [T,d]); idx, gate and slot receive the
 *               per-token results (slot indexes the slice's own buffers);
 *               counts and offsets hold the last slice's.
 *   x_host      [T,d] host (pinned for asynchronous copies)
 *   logits_host [T,E] fp32 host, or NULL when args->logits is NULL
 *   out_host    [T,d] host
 *   stream, stream_h2d, stream_d2h  three distinct streams; when the call
 *               returns, `stream` is ordered after the last copy-out (also
 *               when it returns MOE_ERR_CUDA part-way: then after every copy
 *               it had enqueued).
 * The first call on a device creates the events the pipeline uses (kept
 * for the life of the process); calls from several host threads on one
 * device take turns on them (a per-device lock held while a call enqueues).
 * No save_* buffers in this mode.
 * ---------------------------------------------------------------------- */
MOE_API int moe_layer_fwd_host(const moe_layer_args* args, const void* x_host,
                               const float* logits_host, void* out_host, int chunks,
                               void* stream, void* stream_h2d, void* stream_d2h);

/* ------------------------------------------------------------------------
 * moe_layer_bwd — backward of moe_layer_fwd with the gates held constant:
 *   dYe[slot[t,j]] = bf16(gate[t,j] * dOut[t])       (moe_dispatch, scaled)
 *   moe_grouped_swiglu_bwd                          -> dXe, dW1, dW3, dW2
 *   dx[t] = sum_j dXe[slot[t,j]]                    (moe_combine, unit gates)
 * Needs the forward's routing (slot, gate, offsets) and saved rows (Xe, A,
 * B, H: moe_layer_args.save_*). Workspace: moe_layer_bwd_workspace_size
 * (dYe, dA, dB, dXe). bf16 only, same limits as moe_grouped_swiglu_bwd.
 *
 * With dlogits non-NULL the gates are differentiated too (router backward,
 * see moe_router_bwd): dlogits [T,E] fp32 (and dgate [T,k] if non-NULL)
 * from dOut, the forward's Ye (save_Ye), logits, idx and counts, with
 * aux_coef times the load-balancing loss's gradient; when Wr is given the
 * router GEMM backward follows: dx += dlogits·Wr and, if dWr is non-NULL,
 * dWr = dlogitsᵀ·x ([E,d] bf16, router_workspace of
 * moe_router_linear_bwd_workspace_size bytes).
 * ---------------------------------------------------------------------- */
typedef struct moe_layer_bwd_args {
    int64_t T, d, E, F;
    int32_t k, dtype, reserved0, reserved1;
    const int32_t* slot;    /* [T,k] from the forward                          */
    const float* gate;      /* [T,k]                                          */
    const int32_t* offsets; /* [E+1]                                          */
    const void* Xe;         /* [R,d] saved forward rows                       */
    const void* A;          /* [R,F]                                          */
    const void* B;          /* [R,F]                                          */
    const void* H;          /* [R,F]                                          */
    const void* W1;
    const void* W3;
    const void* W2;
    int64_t w13_expert_stride, w2_expert_stride;
    const void* dOut;       /* [T,d] upstream gradient                        */
    void* dx;               /* [T,d]                                          */
    void* dW1;              /* [E,F,d]                                        */
    void* dW3;              /* [E,F,d]                                        */
    void* dW2;              /* [E,d,F]                                        */
    void* workspace;
    size_t workspace_bytes;
    /* optional router backward (dlogits == NULL: gates held constant) */
    const float* logits;    /* [T,E] fp32 logits of the forward               */
    const int32_t* idx;     /* [T,k]                                          */
    const int32_t* counts;  /* [E]                                            */
    const void* Ye;         /* [R,d] the forward's expert outputs (save_Ye)   */
    const void* x;          /* [T,d] forward input (for dWr)                  */
    const void* Wr;         /* [E,d], or NULL when the logits were an input   */
    float aux_coef;         /* weight of the load-balancing loss              */
    int32_t renorm;         /* the forward's renorm flag                      */
    float* dgate;           /* [T,k] fp32, or NULL                            */
    float* dlogits;         /* [T,E] fp32                                     */
    void* dWr;              /* [E,d], or NULL                                 */
    void* router_workspace;
    size_t router_workspace_bytes;
} moe_layer_bwd_args;

MOE_API size_t moe_layer_bwd_workspace_size(int64_t T, int64_t d, int64_t F, int k, int dtype);
MOE_API int moe_layer_bwd(const moe_layer_bwd_args* args, void* stream);

/* ------------------------------------------------------------------------
 * MXFP8 backward ["专家池 8→128 只慢 5%…", "三招拆分、三项优化、一个精度开关":
 * the MXFP8 switch speeds up training through the FFN and the expert data
 * movement; "olmoforge" README, "MXFP8 分块量化"]. Reading of the backward's
 * precision (the pages leave it open): the two input-gradient GEMMs run on
 * block-scaled FP8 with every operand quantised along its contraction
 * dimension (UE8M0 scales, E4M3 codes), the weight gradients run as bf16
 * GEMMs on the forward's dequantised operands:
 *   dYe[slot[t,j]] = bf16(gate[t,j] * dOut[t])
 *   dH  = Q_d(dYe) · Q_d(W2_e)             (contraction over d)
 *   dA  = dH*B*silu'(A),  dB = dH*silu(A)   (fp32 from bf16 dH, A, B)
 *   dXe = Q_F([dA|dB]) · Q_F([W1_e; W3_e])  (contraction over 2F)
 *   dx[t] = sum_j dXe[slot[t,j]]
 *   dW1_e = dAᵀ·deq(Xq),  dW3_e = dBᵀ·deq(Xq),  dW2_e = dYeᵀ·deq(Hq)
 * with A, B, Xq, Hq the forward's (moe_layer_mxfp8_args.save_*).
 *
 * mxfp8_quantize_weights_bwd: the backward weights, once per weight update.
 *   W1, W3 [E,F,d] and W2 [E,d,F] bf16 (expert strides in elements, rows
 *   contiguous) -> W13tq [E,d,2F] codes with W13ts [E,d,2F/32] scales (row i:
 *   column i of W1_e then column i of W3_e, blocks of 32 along F), and W2tq
 *   [E,F,d] with W2ts [E,F,d/32] (row f: column f of W2_e, blocks along d).
 *   Pack the scales with mxfp8_pack_weight_scales as a W2 operand: W2ts with
 *   (d, F) = (F, d) -> Ps2t, W13ts with (d, F) = (d, 2F) -> Ps13t.
 *   d % 128 == 0, F % 128 == 0; all pointers 16-byte aligned.
 * moe_swiglu_bwd_mxfp8: the SwiGLU backward step alone: dH, A, B [R,F] bf16
 *   -> dA, dB [R,F] bf16 and the codes of [dA|dB] dABq [R,2F] with scales
 *   dABs [R,2F/32] (quantised from the fp32 values). F % 32 == 0.
 * moe_layer_bwd_mxfp8: the whole chain on one stream (moe_dispatch,
 *   mxfp8_quantize, mxfp8_pack_act_scales, moe_grouped_down_mxfp8 for dH
 *   and dXe, moe_swiglu_bwd_mxfp8, moe_combine, mxfp8_dequantize and the
 *   bf16 weight-gradient GEMMs of moe_grouped_swiglu_bwd). d % 256 == 0,
 *   F % 256 == 0. Workspace: moe_layer_bwd_mxfp8_workspace_size bytes,
 *   256-byte aligned. dx [T,d], dW1/dW3 [E,F,d], dW2 [E,d,F] bf16,
 *   contiguous; an expert with no rows gets zero weight gradients. Router
 *   and gate gradients are not part of it (use moe_router_bwd).
 * ---------------------------------------------------------------------- */
MOE_API int mxfp8_quantize_weights_bwd(const void* W1, const void* W3, const void* W2,
                                       int64_t w13_expert_stride, int64_t w2_expert_stride,
                                       int64_t E, int64_t d, int64_t F, uint8_t* W13tq,
                                       uint8_t* W13ts, uint8_t* W2tq, uint8_t* W2ts,
                                       void* stream);
MOE_API int moe_swiglu_bwd_mxfp8(const void* dH, const void* A, const void* B, int64_t R,
                                 int64_t F, void* dA, void* dB, uint8_t* dABq, uint8_t* dABs,
                                 void* stream);

typedef struct moe_layer_bwd_mxfp8_args {
    int64_t T, d, E, F;
    int32_t k, reserved0, reserved1, reserved2;
    const int32_t* slot;    /* [T,k] from the forward                          */
    const float* gate;      /* [T,k]                                          */
    const int32_t* offsets; /* [E+1]                                          */
    const uint8_t* Xq;      /* [R,d] the forward's dispatched codes            */
    const uint8_t* Xs;      /* [R,d/32] their scales, row layout              */
    const uint8_t* Hq;      /* [R,F] the forward's H codes                     */
    const uint8_t* Hsp;     /* H scales, tile-packed (as gate/up wrote them)   */
    const void* A;          /* [R,F] bf16 pre-activations                      */
    const void* B;          /* [R,F] bf16                                      */
    const uint8_t* W13tq;   /* [E,d,2F] (mxfp8_quantize_weights_bwd)           */
    const uint8_t* Ps13t;   /* its packed scales                              */
    const uint8_t* W2tq;    /* [E,F,d]                                        */
    const uint8_t* Ps2t;    /* its packed scales                              */
    const void* dOut;       /* [T,d] bf16 upstream gradient                   */
    void* dx;               /* [T,d] bf16                                     */
    void* dW1;              /* [E,F,d] bf16                                   */
    void* dW3;              /* [E,F,d] bf16                                   */
    void* dW2;              /* [E,d,F] bf16                                   */
    void* workspace;
    size_t workspace_bytes;
} moe_layer_bwd_mxfp8_args;

MOE_API size_t moe_layer_bwd_mxfp8_workspace_size(int64_t T, int64_t d, int64_t E, int64_t F,
                                                  int k);
MOE_API int moe_layer_bwd_mxfp8(const moe_layer_bwd_mxfp8_args* args, void* stream);

/* ------------------------------------------------------------------------
 * Router backward and the load-balancing auxiliary loss.
 *
 * ["Transformers 中的 OLMoE", §2 router; §4 "负载均衡辅助损失": a Switch-
 * Transformer-style loss built from each expert's assignment frequency and
 * its mean routing probability, multiplied and summed; the caller scales it
 * into the total loss (router_aux_loss_coef, 0.01 by default).] p[t,:] is
 * the fp32 softmax of logits[t,:]; f_e = counts[e]/T counts each of a
 * token's k choices (a uniform router gives aux = k).
 *
 * moe_aux_loss: *aux_out (device fp32) = E * sum_e f_e * (1/T) sum_t p[t,e].
 *   logits [T,E] fp32, counts [E] from moe_route. Workspace (16-byte
 *   aligned, moe_aux_loss_workspace_size bytes) holds per-block partial
 *   sums; the result is deterministic (fixed reduction order). T >= 1.
 *
 * moe_router_bwd: gradients of a loss L(out) + aux_coef * aux with respect
 * to the gates and the router logits, the top-k choice and the counts held
 * fixed (both piecewise constant):
 *   dgate[t,j]   = <dOut[t], Ye[slot[t,j]]>   (fp32 sums of the layer-dtype
 *                  rows; out[t] = sum_j gate[t,j] Ye[slot[t,j]])
 *   dsel[t,j]    = dgate, or with renorm (gates p_sel/S, S = sum of the k
 *                  chosen p): (dgate - sum_i gate_i dgate_i) / S
 *   dp[t,e]      = sum_j [idx[t,j] = e] dsel[t,j] + aux_coef*E*counts[e]/T^2
 *   dlogits[t,e] = p[t,e] * (dp[t,e] - sum_e' p[t,e'] dp[t,e'])
 *   dOut [T,d], Ye [R,d] (the forward's expert outputs) in `dtype`, 16-byte
 *   aligned rows; slot, idx [T,k], logits [T,E] fp32 and counts [E] from
 *   the forward (counts may be NULL when aux_coef == 0). dgate [T,k] fp32
 *   (NULL = not written), dlogits [T,E] fp32. A slot or idx out of range is
 *   skipped and sets MOE_DEVERR_BAD_INDEX.
 *
 * moe_router_linear_bwd: the router GEMM logits = x Wr^T:
 *   dx[t,:]  = round(dx[t,:] + sum_e dlogits[t,e] Wr[e,:])  (dx NULL: skip;
 *              accumulates into the layer-dtype dx of moe_layer_bwd)
 *   dWr[e,:] = round(sum_t dlogits[t,e] x[t,:])             (dWr NULL: skip)
 *   fp32 sums (dWr over fixed token chunks, then the chunks in order, in the
 *   workspace of moe_router_linear_bwd_workspace_size bytes). x [T,d],
 *   Wr [E,d], dx, dWr in `dtype`; d % 4 == 0. With bf16 data, d % 256 == 0
 *   and a 256-byte aligned workspace (16-byte aligned x, Wr, dx) the two
 *   products run on the tensor cores, as the bf16 router's backward: dlogits
 *   is rounded to bf16 once and the exact products are summed in fp32;
 *   otherwise on the CUDA cores in fp32 from the fp32 dlogits.
 * ---------------------------------------------------------------------- */
MOE_API size_t moe_aux_loss_workspace_size(int64_t T, int64_t E);
MOE_API int moe_aux_loss(const float* logits, const int32_t* counts, int64_t T, int64_t E,
                         float* aux_out, void* workspace, size_t workspace_bytes, void* stream);
MOE_API int moe_router_bwd(const void* dOut, const void* Ye, const int32_t* slot,
                           const int32_t* idx, const float* logits, const int32_t* counts,
                           int64_t T, int64_t d, int64_t E, int k, int dtype, int renorm,
                           float aux_coef, float* dgate, float* dlogits, void* stream);
MOE_API size_t moe_router_linear_bwd_workspace_size(int64_t T, int64_t d, int64_t E);
MOE_API int moe_router_linear_bwd(const float* dlogits, const void* x, const void* Wr,
                                  int64_t T, int64_t d, int64_t E, int dtype, void* dx,
                                  void* dWr, void* workspace, size_t workspace_bytes,
                                  void* stream);

/* ------------------------------------------------------------------------
 * Expert parallelism over G ranks (one GPU each).
 *
 * ["olmoforge" README, capability table]: row-wise expert parallelism
 * writes every token row straight into the input buffer of its expert, on
 * whichever GPU holds it; [NEWS, "关键数字"]: experts are spread over the GPUs.
 * Rank r owns experts r*El .. (r+1)*El - 1 (El = E / G). Each rank routes its
 * own T tokens with moe_route; the ranks then gather their counts into
 * counts_all [G, E] (row s = rank s's counts, e.g. one all-gather). Rank r's
 * receive buffer holds the rows of its experts expert-major, and within an
 * expert the rows of rank 0, then rank 1, ..., each in its sender's token
 * order; it is the expert-sorted input of rank r's grouped GEMMs with
 * offsets recv_offsets.
 *
 * moe_ep_plan — for this rank (`me`): dst_rank [T,k] and dst_row [T,k], the
 *   owner and the row in the owner's receive buffer of every (t, j), and
 *   recv_offsets [El+1] of this rank's receive buffer (recv_offsets[El] = its
 *   rows). idx, slot, offsets from this rank's moe_route. Workspace:
 *   moe_ep_workspace_size(E) bytes of device memory. Limits: E % G == 0,
 *   1 <= G <= 64. A negative count or an expert index out of range sets
 *   MOE_DEVERR_BAD_INDEX (the row gets dst_rank = dst_row = -1).
 * moe_dispatch_ep — recv_bufs[dst_rank[t,j]][dst_row[t,j], :] = x[t, :].
 *   recv_bufs: device array of G device pointers (8-byte aligned), each a
 *   [rows_max, d] buffer in `dtype`, 16-byte aligned: on a multi-GPU node the
 *   peers' receive buffers mapped into this process, so the rows travel over
 *   NVLink as stores; a row outside [0, rows_max), a null or misaligned
 *   pointer is skipped and sets MOE_DEVERR_BAD_INDEX.
 * moe_combine_ep — out[t] = sum_j gate[t,j] * ye_bufs[dst_rank[t,j]][dst_row[t,j]]
 *   (fp32 fused multiply-add in ascending j, rounded once to `dtype`): the
 *   owners' expert outputs gathered back (peer loads on a multi-GPU node).
 * The caller orders the steps across ranks: every rank's dispatch into a
 * buffer completes before its owner's GEMMs read it, and the owner's GEMMs
 * before any rank's combine reads the output (e.g. a stream-ordered barrier
 * between the steps).
 * ---------------------------------------------------------------------- */
MOE_API size_t moe_ep_workspace_size(int64_t E);
MOE_API int moe_ep_plan(const int32_t* counts_all, int G, int me, const int32_t* idx,
                        const int32_t* slot, const int32_t* offsets, int64_t T, int64_t E, int k,
                        int32_t* dst_rank, int32_t* dst_row, int32_t* recv_offsets,
                        void* workspace, size_t workspace_bytes, void* stream);
MOE_API int moe_dispatch_ep(const void* x, const int32_t* dst_rank, const int32_t* dst_row,
                            int64_t T, int64_t d, int k, int dtype, void* const* recv_bufs, int G,
                            int64_t rows_max, void* stream);
MOE_API int moe_combine_ep(const void* const* ye_bufs, const int32_t* dst_rank,
                           const int32_t* dst_row, const float* gate, int64_t T, int64_t d, int k,
                           int dtype, int G, int64_t rows_max, void* out, void* stream);

/* ------------------------------------------------------------------------
 * moe_get_status — read (and optionally clear) the device status word of the
 * current device. Synchronises the given stream. *host_status receives an OR
 * of MOE_DEVERR_* bits (0 = no fault seen).
 * ---------------------------------------------------------------------- */
MOE_API int moe_get_status(int32_t* host_status, int clear, void* stream);

/* ------------------------------------------------------------------------
 * moe_debug_set_wait_limit_ns — for tests of the fault path only: sets the
 * time limit of every bounded pipeline wait in the tensor-core kernels
 * (grouped GEMMs, backward GEMMs, MXFP8 GEMMs, router) on the current
 * device; 0 restores the default of 2 s. A wait that exceeds the limit sets
 * MOE_DEVERR_TIMEOUT and an abort flag; every role of the kernel then stops
 * issuing, waits (at most 0.1 s) for the copies and MMAs it already has in
 * flight, the tensor memory is freed and the kernel returns with its outputs
 * incomplete. With a limit of a few nanoseconds nearly every wait gives up,
 * which exercises that path without any fault. Synchronous (a copy to device
 * memory); do not change it while kernels of the library are running.
 * ---------------------------------------------------------------------- */
MOE_API int moe_debug_set_wait_limit_ns(uint64_t ns);

/* moe_debug_set_gemm_form — for tests: the tile form of the bf16/fp32
 * grouped GEMMs (moe_grouped_gate_up[_save], moe_grouped_down and the layer
 * entries that call them): 0 = by shape (the default), 1 = row tiles, 2 =
 * token-column tiles wherever the weight layout allows them. Process-wide;
 * MOE_ERR_INVALID for any other value. */
MOE_API int moe_debug_set_gemm_form(int form);

/* library version string */
MOE_API const char* moe_version(void);

#ifdef __cplusplus
}
#endif
#endif /* DROPLESS_TOP_MIXTURE_B200_MOE_H */
