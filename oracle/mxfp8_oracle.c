/*
 * mxfp8_oracle.c -- MXFP8 emulation for the oracle.  TEST INFRASTRUCTURE
 * ONLY (see mok_oracle.c).  Shares nothing with the CUDA path.
 *
 * The MoK article names MXFP8 activation quantisation fused into dispatch,
 * the grouped GEMM and SwiGLU (paragraph after the ring-buffer paragraph),
 * without defining the format.  MXFP8 is the OCP Microscaling format
 * (OCP MX v1.0): blocks of 32 elements share one E8M0 scale X = 2^s, the
 * elements are FP8 E4M3 values P_i and the block represents X * P_i.
 *
 * Conversion of a block (OCP MX v1.0, conversion from a wider type):
 *   s   = floor(log2(max_i |V_i|)) - 8       (8 = exponent of E4M3's
 *                                              largest normal, 448 = 1.75*2^8)
 *   s is clamped to [-127, 127]; an all-zero block gets s = -127.
 *   scale byte = s + 127 (E8M0, bias 127)
 *   P_i = E4M3(V_i / 2^s), round to nearest even, magnitudes above 448
 *         saturate to 448 (the "satfinite" convention), the sign of a value
 *         that rounds to zero is kept.
 * E4M3 (OCP FP8): 1 sign, 4 exponent (bias 7), 3 mantissa bits; no
 * infinities; S.1111.111 is NaN; subnormals m * 2^-9.
 *
 * Everything is done in double / integer arithmetic; the division by 2^s is
 * exact.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_EINVAL 1
#define ORACLE_ENOMEM 2

static double o_bf16(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* round-half-to-even of a non-negative double to an integer */
static double rne(double a) {
    double f = floor(a);
    double d = a - f;
    if (d > 0.5) return f + 1.0;
    if (d < 0.5) return f;
    return (fmod(f, 2.0) == 0.0) ? f : f + 1.0;
}

/* value of an E4M3 byte */
double oracle_e4m3_decode(uint8_t b) {
    int sgn = b >> 7, ex = (b >> 3) & 0xF, m = b & 7;
    double v;
    if (ex == 0xF && m == 7) return NAN;
    if (ex == 0) v = ldexp((double)m, -9);
    else v = ldexp(1.0 + m / 8.0, ex - 7);
    return sgn ? -v : v;
}

/* E4M3 encoding of a finite double, RNE, saturating at 448 */
static uint8_t e4m3_encode(double v) {
    uint8_t sgn = signbit(v) ? 0x80 : 0x00;
    double a = fabs(v);
    if (a >= 448.0) return sgn | 0x7E;                      /* satfinite */
    if (a < ldexp(1.0, -6)) {                               /* subnormal range */
        double q = rne(a / ldexp(1.0, -9));                 /* 0..8 */
        if (q >= 8.0) return sgn | (1 << 3);                /* rounds up to 2^-6 */
        return sgn | (uint8_t)q;
    }
    int e;
    double fr = frexp(a, &e);                                /* a = fr * 2^e, fr in [0.5,1) */
    e -= 1;                                                  /* a = (2 fr) * 2^e */
    double q = rne((2.0 * fr - 1.0) * 8.0);                  /* 0..8 */
    if (q >= 8.0) { q = 0.0; e += 1; }
    if (e > 8 || (e == 8 && q > 6.0)) return sgn | 0x7E;     /* above 448 after rounding */
    return sgn | (uint8_t)(((e + 7) << 3) | (int)q);
}

/* shared exponent s of a block from its largest magnitude */
static int block_exponent(double amax) {
    if (amax == 0.0) return -127;
    int e;
    (void)frexp(amax, &e);
    int s = (e - 1) - 8;
    if (s < -127) s = -127;
    if (s > 127) s = 127;
    return s;
}

/* Quantise n_blocks consecutive blocks of 32 fp32 values. */
int oracle_mxfp8_quantize(const float* v, int64_t n_blocks, uint8_t* q, uint8_t* scales) {
    if (!v || !q || !scales || n_blocks < 0) return ORACLE_EINVAL;
    for (int64_t b = 0; b < n_blocks; ++b) {
        const float* blk = v + b * 32;
        double amax = 0.0;
        for (int i = 0; i < 32; ++i) if (fabs((double)blk[i]) > amax) amax = fabs((double)blk[i]);
        int s = block_exponent(amax);
        scales[b] = (uint8_t)(s + 127);
        for (int i = 0; i < 32; ++i) q[b * 32 + i] = e4m3_encode(ldexp((double)blk[i], -s));
    }
    return ORACLE_OK;
}

/* dequantised copy of a length-n vector (n % 32 == 0) read with stride */
static void mx_roundtrip(const double* src, int n, double* dst) {
    for (int b = 0; b < n / 32; ++b) {
        double amax = 0.0;
        for (int i = 0; i < 32; ++i) if (fabs(src[b * 32 + i]) > amax) amax = fabs(src[b * 32 + i]);
        int s = block_exponent(amax);
        for (int i = 0; i < 32; ++i)
            dst[b * 32 + i] = ldexp(oracle_e4m3_decode(e4m3_encode(ldexp(src[b * 32 + i], -s))), s);
    }
}

/*
 * One expert's SwiGLU FFN on the MXFP8 path (config "page_mxfp8"):
 *   x rows quantised in 32-blocks along H; Wg, Wu quantised in 32-blocks
 *   along their contraction dimension H; Wd along I; the GEMMs use the
 *   dequantised values with exact (double) accumulation; h = silu(a) * b is
 *   rounded to fp32 and quantised in 32-blocks along I before the down
 *   projection.  Optional outputs: h bytes [n, I] and h scales [n, I/32].
 */
int oracle_mxfp8_expert_ffn(const uint16_t* x_rows, int n, int H, int I,
                            const uint16_t* wg, const uint16_t* wu, const uint16_t* wd,
                            double* o, uint8_t* h_q, uint8_t* h_s, void* reserved) {
    (void)reserved;
    if (n < 0 || H <= 0 || I <= 0 || H % 32 || I % 32) return ORACLE_EINVAL;
    if (n == 0) return ORACLE_OK;
    double* qg = (double*)malloc(sizeof(double) * (size_t)H * I);   /* [I][H]: column i over K=H */
    double* qu = (double*)malloc(sizeof(double) * (size_t)H * I);
    double* qd = (double*)malloc(sizeof(double) * (size_t)I * H);   /* [H][I]: column c over K=I */
    int rc = ORACLE_OK;
    if (!qg || !qu || !qd) {
        free(qg); free(qu); free(qd);
        return ORACLE_ENOMEM;
    }
    /* Columns and rows are independent; threads split them and each element
     * is computed exactly as in a serial run. */
#pragma omp parallel
    {
        double* col = (double*)malloc(sizeof(double) * (size_t)(H > I ? H : I));
        double* xr = (double*)malloc(sizeof(double) * (size_t)H);
        double* xq = (double*)malloc(sizeof(double) * (size_t)H);
        double* hv = (double*)malloc(sizeof(double) * (size_t)I);
        double* hq = (double*)malloc(sizeof(double) * (size_t)I);
        float* hf = (float*)malloc(sizeof(float) * (size_t)I);
        const int ok = col && xr && xq && hv && hq && hf;
        if (!ok) {
#pragma omp atomic write
            rc = ORACLE_ENOMEM;
        }
        /* weights: blocks along the contraction index of each output column */
#pragma omp for schedule(static)
        for (int i = 0; i < I; ++i) {
            if (!ok) continue;
            for (int k = 0; k < H; ++k) col[k] = o_bf16(wg[(size_t)k * I + i]);
            mx_roundtrip(col, H, qg + (size_t)i * H);
            for (int k = 0; k < H; ++k) col[k] = o_bf16(wu[(size_t)k * I + i]);
            mx_roundtrip(col, H, qu + (size_t)i * H);
        }
#pragma omp for schedule(static)
        for (int c = 0; c < H; ++c) {
            if (!ok) continue;
            for (int k = 0; k < I; ++k) col[k] = o_bf16(wd[(size_t)k * H + c]);
            mx_roundtrip(col, I, qd + (size_t)c * I);
        }
#pragma omp for schedule(dynamic, 1)
        for (int r = 0; r < n; ++r) {
            if (!ok) continue;
            for (int k = 0; k < H; ++k) xr[k] = o_bf16(x_rows[(size_t)r * H + k]);
            mx_roundtrip(xr, H, xq);
            for (int i = 0; i < I; ++i) {
                double a = 0.0, b = 0.0;
                const double* g = qg + (size_t)i * H;
                const double* u = qu + (size_t)i * H;
                for (int k = 0; k < H; ++k) { a += xq[k] * g[k]; b += xq[k] * u[k]; }
                hf[i] = (float)(a / (1.0 + exp(-a)) * b);
            }
            if (h_q && h_s) oracle_mxfp8_quantize(hf, I / 32, h_q + (size_t)r * I, h_s + (size_t)r * (I / 32));
            for (int i = 0; i < I; ++i) hv[i] = (double)hf[i];
            mx_roundtrip(hv, I, hq);
            for (int c = 0; c < H; ++c) {
                double acc = 0.0;
                const double* d = qd + (size_t)c * I;
                for (int i = 0; i < I; ++i) acc += hq[i] * d[i];
                o[(size_t)r * H + c] = acc;
            }
        }
        free(col); free(xr); free(xq); free(hv); free(hq); free(hf);
    }
    free(qg); free(qu); free(qd);
    return rc;
}
