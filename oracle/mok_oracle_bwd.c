/*
 * mok_oracle_bwd.c -- plain CPU oracle of the BACKWARD pass of the
 * Mixture-of-Kittens MoE layer.  TEST INFRASTRUCTURE ONLY (see
 * mok_oracle.c): the test suite is its only user, and it shares nothing with
 * the CUDA path.
 *
 * Source: MoK article (tahou.com), the paragraph on Pull and Push: the
 * forward pairs pull dispatch with push combine, and the backward pairs the
 * reverse of each -- a pull reverse-combine (the expert side reads the
 * output gradient of each token it served) and a push reverse-dispatch (the
 * input gradient of each row goes straight back to its token).  The pages
 * give the data movement only; the arithmetic below is the derivative of the
 * forward layer that mok_oracle.c defines (a plain reading: the backward of
 * a layer is its chain rule), in the pages' order of steps:
 *
 *   forward, per token t and rank j with expert e = sel[t, j]:
 *     a = x_t Wg[e],  b = x_t Wu[e],  h = silu(a) * b,  o_tj = h Wd[e]
 *     g_t = softmax over the k selected logits,  y_t = sum_j g_tj o_tj
 *   backward, given dy:
 *     1. pull reverse-combine: for the row of (t, j)
 *          do_tj = g_tj dy_t               (the row's output gradient)
 *          dg_tj = <dy_t, o_tj>            (the gate's gradient)
 *     2. expert FFN backward on the row:
 *          dh = do Wd[e]^T,  dWd[e] += h^T do
 *          da = dh * b * silu'(a),  db = dh * silu(a)
 *          silu'(a) = s + a s (1 - s),  s = 1 / (1 + exp(-a))
 *          dWg[e] += x_t^T da,  dWu[e] += x_t^T db
 *          dx_row = da Wg[e]^T + db Wu[e]^T
 *     3. push reverse-dispatch: dx_t += dx_row of each of its k rows
 *     4. gates: softmax backward over the k selected logits,
 *          dl_tj = g_tj (dg_tj - sum_i g_ti dg_ti),
 *        scattered to dlogits[t, sel[t, j]]; unselected logits get 0 (the
 *        top-k selection itself has no gradient).
 *
 * Everything is double precision, with the gates recomputed in double (not
 * the fp32 gates the forward oracle returns), so the result is the exact
 * derivative up to rounding.  Row order, schedule and gather are the
 * forward oracle's (expert-major rows, ascending tokens inside an expert).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_EINVAL 1
#define ORACLE_ENOMEM 2

int oracle_topk_gates(const float* logits, int T, int E, int k, int32_t* topk_idx, float* gates);
int oracle_schedule(const int32_t* topk_idx, int T, int E, int k, int R, int32_t* counts, int32_t* offsets,
                    int32_t* src_rank, int32_t* src_index, int32_t* row_slot, int32_t* pos);

static double b2d(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/*
 * x [T, H] bf16, logits [T, E] fp32, wg/wu [E, H, I] bf16, wd [E, I, H] bf16,
 * dy [T, H] double.  Outputs (double, overwritten): dx [T, H], dwg/dwu
 * [E, H, I], dwd [E, I, H], dlogits [T, E].
 */
int oracle_moe_backward(const uint16_t* x, const float* logits, int T, int H, int I, int E, int k, int R,
                        const uint16_t* wg, const uint16_t* wu, const uint16_t* wd, const double* dy,
                        double* dx, double* dwg, double* dwu, double* dwd, double* dlogits) {
    if (!x || !logits || !wg || !wu || !wd || !dy || !dx || !dwg || !dwu || !dwd || !dlogits || T <= 0 ||
        H <= 0 || I <= 0 || E <= 0 || k <= 0 || k > E || R <= 0 || T % R != 0)
        return ORACLE_EINVAL;
    const size_t NS = (size_t)T * k;
    int32_t* topk = (int32_t*)malloc(sizeof(int32_t) * NS);
    float* gates32 = (float*)malloc(sizeof(float) * NS);
    double* g = (double*)malloc(sizeof(double) * NS);
    double* dg = (double*)malloc(sizeof(double) * NS);
    int32_t* counts = (int32_t*)malloc(sizeof(int32_t) * (size_t)E);
    int32_t* offsets = (int32_t*)malloc(sizeof(int32_t) * ((size_t)E + 1));
    int32_t* rslot = (int32_t*)malloc(sizeof(int32_t) * NS);
    double* xr = (double*)malloc(sizeof(double) * (size_t)H);
    double* a = (double*)malloc(sizeof(double) * (size_t)I);
    double* b = (double*)malloc(sizeof(double) * (size_t)I);
    double* h = (double*)malloc(sizeof(double) * (size_t)I);
    double* dh = (double*)malloc(sizeof(double) * (size_t)I);
    double* da = (double*)malloc(sizeof(double) * (size_t)I);
    double* db = (double*)malloc(sizeof(double) * (size_t)I);
    double* o = (double*)malloc(sizeof(double) * (size_t)H);
    double* dout = (double*)malloc(sizeof(double) * (size_t)H);
    int rc = ORACLE_ENOMEM;
    if (!topk || !gates32 || !g || !dg || !counts || !offsets || !rslot || !xr || !a || !b || !h || !dh || !da ||
        !db || !o || !dout)
        goto done;
    /* selection and schedule exactly as the forward */
    rc = oracle_topk_gates(logits, T, E, k, topk, gates32);
    if (rc) goto done;
    rc = oracle_schedule(topk, T, E, k, R, counts, offsets, NULL, NULL, rslot, NULL);
    if (rc) goto done;
    /* gates in double: softmax over the selected logits (the first is the largest) */
    for (int t = 0; t < T; ++t) {
        const float* l = logits + (size_t)t * E;
        const double m = (double)l[topk[(size_t)t * k]];
        double s = 0.0;
        for (int j = 0; j < k; ++j) s += exp((double)l[topk[(size_t)t * k + j]] - m);
        for (int j = 0; j < k; ++j) g[(size_t)t * k + j] = exp((double)l[topk[(size_t)t * k + j]] - m) / s;
    }
    memset(dx, 0, sizeof(double) * (size_t)T * H);
    memset(dwg, 0, sizeof(double) * (size_t)E * H * I);
    memset(dwu, 0, sizeof(double) * (size_t)E * H * I);
    memset(dwd, 0, sizeof(double) * (size_t)E * I * H);
    memset(dlogits, 0, sizeof(double) * (size_t)T * E);
    /* rows in expert-major order: steps 1-3 per row */
    for (int e = 0; e < E; ++e) {
        const uint16_t* Wg = wg + (size_t)e * H * I;
        const uint16_t* Wu = wu + (size_t)e * H * I;
        const uint16_t* Wd = wd + (size_t)e * I * H;
        double* dWg = dwg + (size_t)e * H * I;
        double* dWu = dwu + (size_t)e * H * I;
        double* dWd = dwd + (size_t)e * I * H;
        for (int row = offsets[e]; row < offsets[e + 1]; ++row) {
            const int slot = rslot[row];
            const int t = slot / k;
            /* recompute the row's forward: a, b, h, o */
            for (int c = 0; c < H; ++c) xr[c] = b2d(x[(size_t)t * H + c]);
            for (int i = 0; i < I; ++i) { a[i] = 0.0; b[i] = 0.0; }
            for (int c = 0; c < H; ++c)
                for (int i = 0; i < I; ++i) {
                    a[i] += xr[c] * b2d(Wg[(size_t)c * I + i]);
                    b[i] += xr[c] * b2d(Wu[(size_t)c * I + i]);
                }
            for (int i = 0; i < I; ++i) h[i] = a[i] / (1.0 + exp(-a[i])) * b[i];
            for (int c = 0; c < H; ++c) o[c] = 0.0;
            for (int i = 0; i < I; ++i)
                for (int c = 0; c < H; ++c) o[c] += h[i] * b2d(Wd[(size_t)i * H + c]);
            /* 1. pull reverse-combine */
            const double* dyt = dy + (size_t)t * H;
            double dgs = 0.0;
            for (int c = 0; c < H; ++c) {
                dout[c] = g[slot] * dyt[c];
                dgs += dyt[c] * o[c];
            }
            dg[slot] = dgs;
            /* 2. expert FFN backward */
            for (int i = 0; i < I; ++i) {
                double acc = 0.0;
                for (int c = 0; c < H; ++c) acc += dout[c] * b2d(Wd[(size_t)i * H + c]);
                dh[i] = acc;
                for (int c = 0; c < H; ++c) dWd[(size_t)i * H + c] += h[i] * dout[c];
            }
            for (int i = 0; i < I; ++i) {
                const double s = 1.0 / (1.0 + exp(-a[i]));
                da[i] = dh[i] * b[i] * (s + a[i] * s * (1.0 - s));
                db[i] = dh[i] * a[i] * s;
            }
            for (int c = 0; c < H; ++c) {
                double acc = 0.0;
                for (int i = 0; i < I; ++i) {
                    dWg[(size_t)c * I + i] += xr[c] * da[i];
                    dWu[(size_t)c * I + i] += xr[c] * db[i];
                    acc += da[i] * b2d(Wg[(size_t)c * I + i]) + db[i] * b2d(Wu[(size_t)c * I + i]);
                }
                /* 3. push reverse-dispatch: the row's input gradient goes back to its token */
                dx[(size_t)t * H + c] += acc;
            }
        }
    }
    /* 4. softmax backward over each token's k selected logits */
    for (int t = 0; t < T; ++t) {
        double dot = 0.0;
        for (int j = 0; j < k; ++j) dot += g[(size_t)t * k + j] * dg[(size_t)t * k + j];
        for (int j = 0; j < k; ++j)
            dlogits[(size_t)t * E + topk[(size_t)t * k + j]] = g[(size_t)t * k + j] * (dg[(size_t)t * k + j] - dot);
    }
    rc = ORACLE_OK;
done:
    free(topk); free(gates32); free(g); free(dg); free(counts); free(offsets); free(rslot);
    free(xr); free(a); free(b); free(h); free(dh); free(da); free(db); free(o); free(dout);
    return rc;
}
