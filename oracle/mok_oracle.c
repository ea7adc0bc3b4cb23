/*
 * mok_oracle.c -- plain, slow CPU oracle of the Mixture-of-Kittens forward
 * MoE layer.  TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and
 * the benchmark's CPU-baseline leg are the only users.  It shares no code,
 * header, table or helper with the CUDA path under combine_device_top_b200/.
 *
 * What the layer computes (sources):
 *  - "MoK article" = tahou.com article on Mixture-of-Kittens (summary +
 *    body).  The routing paragraph: the router assigns each token to
 *    experts; the system counts the tokens of every expert, plans where they
 *    go and lays tokens of one expert out contiguously so that a grouped GEMM
 *    can run on them.  The pull paragraph: the destination reads what it
 *    needs knowing only the source rank and the offset there.  The
 *    push-combine paragraph: each expert result goes back to its token's
 *    slot.  The benchmark paragraph: the layer ends with a weighted merge.
 *  - "MoK wiki summary" = "Mixture-of-Kittens: Cursor가 새로 공개한 NVL72용 MoE
 *    학습 메가커널" (LLM Wiki), key points: the schedule is a table of
 *    {src_rank, src_index} built on the device with no sort.
 *
 * Readings where the pages are silent (each is stated again beside the code):
 *  - gates: softmax over the k selected logits;
 *  - ties in top-k: the lower expert index wins;
 *  - order of rows inside an expert segment: ascending token index;
 *  - slot j of a token: its rank in the top-k list;
 *  - expert FFN: SwiGLU, h = silu(x Wg) * (x Wu), o = h Wd;
 *  - combine: y[t] = sum_j g[t,j] o[t,j], j ascending;
 *  - shard r holds tokens [r*S_r, (r+1)*S_r), S_r = T / R.
 *
 * Arithmetic is in double precision throughout; bf16 inputs are widened
 * exactly.  Nothing is rounded to bf16 inside the layer here.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_EINVAL 1
#define ORACLE_ENOMEM 2

/* bf16 bit pattern -> exact double. */
static double bf16_to_double(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* ------------------------------------------------------------------------
 * Step 1: router top-k and gates (MoK article, routing paragraph).
 * For every token the selected list is the first k experts in the order
 * (logit descending, expert index ascending).  Gates are the softmax of the
 * k selected logits.  Written as k rounds of "pick the best remaining
 * expert", which is the definition of that order's first k elements.
 * ---------------------------------------------------------------------- */
int oracle_topk_gates(const float* logits, int T, int E, int k,
                      int32_t* topk_idx, float* gates) {
    if (!logits || !topk_idx || !gates || T < 0 || E <= 0 || k <= 0 || k > E) return ORACLE_EINVAL;
    unsigned char* taken = (unsigned char*)malloc((size_t)E);
    double* ex = (double*)malloc(sizeof(double) * (size_t)k);
    if (!taken || !ex) { free(taken); free(ex); return ORACLE_ENOMEM; }
    for (int t = 0; t < T; ++t) {
        const float* l = logits + (size_t)t * E;
        memset(taken, 0, (size_t)E);
        for (int j = 0; j < k; ++j) {
            int best = -1;
            for (int e = 0; e < E; ++e) {
                if (taken[e]) continue;
                /* strictly greater: an equal logit at a higher index loses */
                if (best < 0 || l[e] > l[best]) best = e;
            }
            taken[best] = 1;
            topk_idx[(size_t)t * k + j] = best;
        }
        /* softmax over the selected logits; the first one is the maximum */
        double m = (double)l[topk_idx[(size_t)t * k]];
        double s = 0.0;
        for (int j = 0; j < k; ++j) {
            ex[j] = exp((double)l[topk_idx[(size_t)t * k + j]] - m);
            s += ex[j];
        }
        for (int j = 0; j < k; ++j) gates[(size_t)t * k + j] = (float)(ex[j] / s);
    }
    free(taken);
    free(ex);
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------
 * Step 2: counts, offsets and the pull schedule (MoK article, routing and
 * pull paragraphs; MoK wiki summary, schedule bullet).
 *   counts[e]   = number of (t, j) with topk_idx[t, j] == e
 *   offsets     = exclusive prefix sum of counts, offsets[E] = T*k
 *   rows of expert e are offsets[e] .. offsets[e+1]-1, tokens ascending;
 *   for the row of (t, j):  src_rank = t / S_r,  src_index = t % S_r,
 *   row_slot = t*k + j, and pos[t*k + j] = row.
 * Written as the plain two-pass counting placement: count, then walk the
 * experts and, inside each, the tokens in order.
 * ---------------------------------------------------------------------- */
int oracle_schedule(const int32_t* topk_idx, int T, int E, int k, int R,
                    int32_t* counts, int32_t* offsets,
                    int32_t* src_rank, int32_t* src_index,
                    int32_t* row_slot, int32_t* pos) {
    if (!topk_idx || !counts || !offsets || T < 0 || E <= 0 || k <= 0 || R <= 0 || T % R != 0)
        return ORACLE_EINVAL;
    const int S_r = T / R;
    for (int e = 0; e < E; ++e) counts[e] = 0;
    for (size_t s = 0; s < (size_t)T * k; ++s) {
        int e = topk_idx[s];
        if (e < 0 || e >= E) return ORACLE_EINVAL;
        counts[e]++;
    }
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
    for (int e = 0; e < E; ++e) {
        int next = offsets[e];
        for (int t = 0; t < T; ++t) {
            for (int j = 0; j < k; ++j) {
                if (topk_idx[(size_t)t * k + j] != e) continue;
                int row = next++;
                if (src_rank) src_rank[row] = t / S_r;
                if (src_index) src_index[row] = t % S_r;
                if (row_slot) row_slot[row] = t * k + j;
                if (pos) pos[(size_t)t * k + j] = row;
            }
        }
    }
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------
 * Step 3: pull dispatch = gather (MoK article, pull paragraph).  Row `row`
 * of the expert-major layout is token src_index of shard src_rank.  A copy.
 * ---------------------------------------------------------------------- */
int oracle_gather(const uint16_t* x, int T, int H, int R, int n_rows,
                  const int32_t* src_rank, const int32_t* src_index, uint16_t* rows) {
    if (!x || !rows || T <= 0 || H <= 0 || R <= 0 || T % R != 0) return ORACLE_EINVAL;
    const int S_r = T / R;
    for (int row = 0; row < n_rows; ++row) {
        int r = src_rank[row], i = src_index[row];
        if (r < 0 || r >= R || i < 0 || i >= S_r) return ORACLE_EINVAL;
        const uint16_t* shard = x + (size_t)r * S_r * H;   /* shard r's own base */
        memcpy(rows + (size_t)row * H, shard + (size_t)i * H, sizeof(uint16_t) * (size_t)H);
    }
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------
 * Step 4: one expert's SwiGLU FFN on n rows (MoK article: grouped GEMM of
 * the expert FFN; SwiGLU named where the MXFP8 fusion is described).
 *   a = x Wg, b = x Wu           (Wg, Wu: [H, I] row-major)
 *   h_i = a_i / (1 + exp(-a_i)) * b_i
 *   o = h Wd                      (Wd: [I, H] row-major)
 * Double accumulation, sums over the contraction index in ascending order.
 * ---------------------------------------------------------------------- */
int oracle_expert_ffn(const uint16_t* x_rows, int n, int H, int I,
                      const uint16_t* wg, const uint16_t* wu, const uint16_t* wd,
                      double* o) {
    if (n < 0 || H <= 0 || I <= 0 || (n > 0 && (!x_rows || !wg || !wu || !wd || !o))) return ORACLE_EINVAL;
    int err = ORACLE_OK;
#pragma omp parallel
    {
        double* a = (double*)malloc(sizeof(double) * (size_t)I);
        double* b = (double*)malloc(sizeof(double) * (size_t)I);
        if (!a || !b) {
#pragma omp atomic write
            err = ORACLE_ENOMEM;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int r = 0; r < n; ++r) {
                const uint16_t* xr = x_rows + (size_t)r * H;
                for (int i = 0; i < I; ++i) { a[i] = 0.0; b[i] = 0.0; }
                for (int hh = 0; hh < H; ++hh) {
                    double xv = bf16_to_double(xr[hh]);
                    const uint16_t* g = wg + (size_t)hh * I;
                    const uint16_t* u = wu + (size_t)hh * I;
                    for (int i = 0; i < I; ++i) {
                        a[i] += xv * bf16_to_double(g[i]);
                        b[i] += xv * bf16_to_double(u[i]);
                    }
                }
                for (int i = 0; i < I; ++i) a[i] = a[i] / (1.0 + exp(-a[i])) * b[i];  /* h */
                double* orow = o + (size_t)r * H;
                for (int c = 0; c < H; ++c) orow[c] = 0.0;
                for (int i = 0; i < I; ++i) {
                    double hv = a[i];
                    const uint16_t* d = wd + (size_t)i * H;
                    for (int c = 0; c < H; ++c) orow[c] += hv * bf16_to_double(d[c]);
                }
            }
        }
        free(a);
        free(b);
    }
    return err;
}

/* ------------------------------------------------------------------------
 * Step 5: combine = weighted merge (MoK article, benchmark paragraph; push
 * combine paragraph).  y[t] = sum_{j=0}^{k-1} g[t,j] * o[t,j], j ascending.
 * o_slot is indexed by slot t*k + j.
 * ---------------------------------------------------------------------- */
int oracle_combine(const double* o_slot, const float* gates, int T, int k, int H, double* y) {
    if (!o_slot || !gates || !y || T < 0 || k <= 0 || H <= 0) return ORACLE_EINVAL;
    for (int t = 0; t < T; ++t) {
        double* yr = y + (size_t)t * H;
        for (int c = 0; c < H; ++c) yr[c] = 0.0;
        for (int j = 0; j < k; ++j) {
            double g = (double)gates[(size_t)t * k + j];
            const double* orow = o_slot + ((size_t)t * k + j) * H;
            for (int c = 0; c < H; ++c) yr[c] += g * orow[c];
        }
    }
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------
 * The whole layer on small inputs: steps 1..5 in the pages' order.
 * x: [T, H] bf16 (shards concatenated), logits [T, E] fp32,
 * wg/wu: [E, H, I] bf16, wd: [E, I, H] bf16.  y: [T, H] double.
 * Optional outputs (may be NULL): topk_idx, gates [T*k].
 * ---------------------------------------------------------------------- */
int oracle_moe_forward(const uint16_t* x, const float* logits,
                       int T, int H, int I, int E, int k, int R,
                       const uint16_t* wg, const uint16_t* wu, const uint16_t* wd,
                       double* y, int32_t* topk_out, float* gates_out) {
    if (!x || !logits || !wg || !wu || !wd || !y || T <= 0 || H <= 0 || I <= 0 || E <= 0 ||
        k <= 0 || k > E || R <= 0 || T % R != 0)
        return ORACLE_EINVAL;
    const size_t NS = (size_t)T * k;
    int32_t* topk = (int32_t*)malloc(sizeof(int32_t) * NS);
    float* gates = (float*)malloc(sizeof(float) * NS);
    int32_t* counts = (int32_t*)malloc(sizeof(int32_t) * (size_t)E);
    int32_t* offsets = (int32_t*)malloc(sizeof(int32_t) * ((size_t)E + 1));
    int32_t* srank = (int32_t*)malloc(sizeof(int32_t) * NS);
    int32_t* sidx = (int32_t*)malloc(sizeof(int32_t) * NS);
    int32_t* rslot = (int32_t*)malloc(sizeof(int32_t) * NS);
    uint16_t* rows = (uint16_t*)malloc(sizeof(uint16_t) * NS * (size_t)H);
    double* o_row = (double*)malloc(sizeof(double) * NS * (size_t)H);
    double* o_slot = (double*)malloc(sizeof(double) * NS * (size_t)H);
    int rc = ORACLE_ENOMEM;
    if (!topk || !gates || !counts || !offsets || !srank || !sidx || !rslot || !rows || !o_row || !o_slot)
        goto done;
    rc = oracle_topk_gates(logits, T, E, k, topk, gates);
    if (rc) goto done;
    rc = oracle_schedule(topk, T, E, k, R, counts, offsets, srank, sidx, rslot, NULL);
    if (rc) goto done;
    rc = oracle_gather(x, T, H, R, (int)NS, srank, sidx, rows);
    if (rc) goto done;
    for (int e = 0; e < E && !rc; ++e) {
        int r0 = offsets[e], n = counts[e];
        rc = oracle_expert_ffn(rows + (size_t)r0 * H, n, H, I,
                               wg + (size_t)e * H * I, wu + (size_t)e * H * I, wd + (size_t)e * I * H,
                               o_row + (size_t)r0 * H);
    }
    if (rc) goto done;
    /* push combine: row results go back to their token slot */
    for (size_t row = 0; row < NS; ++row)
        memcpy(o_slot + (size_t)rslot[row] * H, o_row + row * H, sizeof(double) * (size_t)H);
    rc = oracle_combine(o_slot, gates, T, k, H, y);
    if (!rc && topk_out) memcpy(topk_out, topk, sizeof(int32_t) * NS);
    if (!rc && gates_out) memcpy(gates_out, gates, sizeof(float) * NS);
done:
    free(topk); free(gates); free(counts); free(offsets); free(srank); free(sidx); free(rslot);
    free(rows); free(o_row); free(o_slot);
    return rc;
}
