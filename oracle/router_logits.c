/*
 * CPU oracle — TEST INFRASTRUCTURE ONLY. Nothing in the product path may
 * call, link or load this file; only the test-suite, the smoke check and the
 * CPU-baseline leg of the benchmark do.
 *
 * Router logits of the dropless top-k MoE layer.
 *
 * The router is a bias-free linear map with a weight of shape
 * (num_experts, hidden_size): logits = x · Wrᵀ ("Transformers 中的 OLMoE",
 * blog.gitcode.com, section 2 "路由器：softmax + top-k 的 token 级路由").
 *
 * The pages leave the summation order of this dot product open. Because the
 * top-k decision is taken on these fp32 values, both sides must produce the
 * same bits, so the order is fixed to the plainest one: one fp32 accumulator
 * per (token, expert), started at +0.0 and updated with a fused multiply-add
 * for j = 0, 1, ..., d-1 in ascending order:
 *
 *     acc <- fmaf(x[t][j], Wr[e][j], acc)
 *
 * (For bf16 inputs the product is exact in fp32, so this equals the unfused
 * acc + x*w; for fp32 inputs the single rounding of fmaf is what is meant.)
 *
 * Built with -ffp-contract=off so the compiler introduces no other fusion.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

/* bf16 -> fp32 is exact: the 16 stored bits are the high half of the fp32. */
static float bf16_to_f32(uint16_t h) {
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* logits[t*E + e] for x [T,d] and Wr [E,d], both fp32, row-major. */
void oracle_router_logits_f32(const float *x, const float *Wr, int64_t T, int64_t d,
                              int64_t E, float *logits) {
    #pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t e = 0; e < E; ++e) {
            float acc = 0.0f;
            for (int64_t j = 0; j < d; ++j)
                acc = fmaf(x[t * d + j], Wr[e * d + j], acc);
            logits[t * E + e] = acc;
        }
    }
}

/* Same, for bf16 x and Wr given as raw 16-bit patterns. */
void oracle_router_logits_bf16(const uint16_t *x, const uint16_t *Wr, int64_t T, int64_t d,
                               int64_t E, float *logits) {
    #pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t e = 0; e < E; ++e) {
            float acc = 0.0f;
            for (int64_t j = 0; j < d; ++j)
                acc = fmaf(bf16_to_f32(x[t * d + j]), bf16_to_f32(Wr[e * d + j]), acc);
            logits[t * E + e] = acc;
        }
    }
}
