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
 * same bits, so the order is fixed: d is cut into four contiguous quarters
 * (d % 4 == 0); in each quarter one fp32 accumulator starts at +0.0 and is
 * updated with a fused multiply-add for j ascending, and the four quarter
 * sums are added in order:
 *
 *     c_q    = fmaf-chain over j in [q d/4, (q+1) d/4):  acc <- fmaf(x, w, acc)
 *     logit  = ((c_0 + c_1) + c_2) + c_3
 *
 * (Four independent chains per logit give the GPU four times the parallel
 * work of a single chain; for bf16 inputs each product is exact in fp32, so
 * fmaf equals the unfused acc + x*w; for fp32 inputs the single rounding of
 * fmaf is what is meant.)
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
    const int64_t dq = d / 4;
    #pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t e = 0; e < E; ++e) {
            float sum = 0.0f;
            for (int q = 0; q < 4; ++q) {
                float acc = 0.0f;
                for (int64_t j = q * dq; j < (q + 1) * dq; ++j)
                    acc = fmaf(x[t * d + j], Wr[e * d + j], acc);
                sum = q == 0 ? acc : sum + acc;
            }
            logits[t * E + e] = sum;
        }
    }
}

/* Same, for bf16 x and Wr given as raw 16-bit patterns. */
void oracle_router_logits_bf16(const uint16_t *x, const uint16_t *Wr, int64_t T, int64_t d,
                               int64_t E, float *logits) {
    const int64_t dq = d / 4;
    #pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t e = 0; e < E; ++e) {
            float sum = 0.0f;
            for (int q = 0; q < 4; ++q) {
                float acc = 0.0f;
                for (int64_t j = q * dq; j < (q + 1) * dq; ++j)
                    acc = fmaf(bf16_to_f32(x[t * d + j]), bf16_to_f32(Wr[e * d + j]), acc);
                sum = q == 0 ? acc : sum + acc;
            }
            logits[t * E + e] = sum;
        }
    }
}
