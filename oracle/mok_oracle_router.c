/*
 * mok_oracle_router.c -- the router projection, for the next row of the
 * path (an on-device router GEMM fused with the top-k).  TEST
 * INFRASTRUCTURE ONLY (see mok_oracle.c); shares nothing with the CUDA path.
 *
 * MoK article (tahou.com), routing paragraph: a router module assigns every
 * token to its experts.  The pages give no formula; the plain reading,
 * which the forward's inputs already follow, is a linear projection of the
 * token onto one logit per expert, plus an optional per-expert bias (the
 * skewed-routing workload adds a log Zipf prior there):
 *     logits[t, e] = sum_h x[t, h] W_r[h, e] + prior[e]
 * x is bf16 [T, H], W_r fp32 [H, E], prior fp32 [E] or NULL; the result is
 * double, summed over h in ascending order.
 */
#include <stdint.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_EINVAL 1

static double r_bf16(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

int oracle_router_logits(const uint16_t* x, const float* wr, const float* prior, int T, int H, int E,
                         double* logits) {
    if (!x || !wr || !logits || T < 0 || H <= 0 || E <= 0) return ORACLE_EINVAL;
    for (int t = 0; t < T; ++t) {
        double* out = logits + (size_t)t * E;
        for (int e = 0; e < E; ++e) out[e] = prior ? (double)prior[e] : 0.0;
        for (int h = 0; h < H; ++h) {
            const double xv = r_bf16(x[(size_t)t * H + h]);
            const float* w = wr + (size_t)h * E;
            for (int e = 0; e < E; ++e) out[e] += xv * (double)w[e];
        }
    }
    return ORACLE_OK;
}
