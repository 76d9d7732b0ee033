/*
 * svdq_oracle.c -- plain, slow CPU oracle for the SVDQuant W4A4 + low-rank
 * linear layer.
 *
 * TEST INFRASTRUCTURE.  Only the tests, the smoke check and the CPU-baseline
 * leg of the benchmark may load this file's library.  It shares no code,
 * header, table or constant with the CUDA library; every number format is
 * decoded from its bit-field definition and every rounding is a search for
 * the nearest representable value, so each step can be checked by eye.
 *
 * Source: "SVDQuant: Absorbing Outliers by Low-Rank Components for 4-Bit
 * Diffusion Models" (arXiv 2411.05007):
 *   Sec. 3 "Quantization Preliminary": Q_X = round(X / s_X), s_X = max|X| / q_max,
 *        q_max = 7 for signed 4-bit integers, 6 for FP4 with 2 exponent bits and
 *        1 mantissa bit; dequantized value s_X * Q_X; XW ~ s_X s_W Q_X Q_W.
 *   Sec. 4.2 "SVDQuant": X_hat = X diag(lambda)^-1, W_hat = diag(lambda) W,
 *        X W ~ X_hat L1 L2 + Q(X_hat) Q(R), low-rank branch in 16 bits.
 *   Sec. 5.1 "Implementation details": per-group symmetric quantization of both
 *        operands; INT4 uses groups of 64 with 16-bit scales; FP4 uses groups of
 *        32 with an FP8 scale.  Three formats are built: NVFP4 (E2M1 codes, one
 *        E4M3 scale per 16 values), FP4 g32 (E2M1 codes, one E4M3 scale per 32
 *        values: the paper's FP4, FP8 read as E4M3) and INT4 (groups of 64).
 *
 * Readings of steps the paper leaves open:
 *   - groups run along K, the reduction dimension, for both operands;
 *   - the scale is amax / q_max computed in fp32 (IEEE division), then rounded
 *     to the scale format (E4M3 saturating / fp16 saturating, nearest-even);
 *   - X / s is computed as X * RN(1/s) in fp32 (the decision is taken in fp32);
 *   - codes round to nearest, ties to the even code; a zero scale gives zero
 *     codes; the sign bit of an E2M1 code is the sign of X * RN(1/s);
 *   - INT4 codes are clamped to [-7, 7] (symmetric, q_max = 7);
 *   - the down-projection is X_hat L1 itself: x_hat = fp32(x) * inv_lambda
 *     (the value the quantizer sees) times the bf16 factor L1, accumulated in
 *     fp32 in increasing k; the branch's intermediate X_hat L1 stays at fp32
 *     accumulator precision (only the factors L1, L2 are 16-bit);
 *   - the GEMM accumulates in fp32: exact per-group integer/E2M1 partial sums,
 *     scaled by s_x * s_w, summed over groups in increasing order, then the
 *     low-rank term sum_j XL1[m,j] L2[j,n] in increasing j, then the bias.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define ORACLE_NVFP4 0
#define ORACLE_INT4 1
#define ORACLE_FP4G32 2
/* W8A8 (the paper's 8-bit setting) has its own functions below: int8 codes one
 * per byte, one fp32 scale per token row (activations) or per output channel
 * (weights), taken over the whole of K. */

/* Group size along K and bytes per scale of each format. */
static int fmt_group(int fmt) { return fmt == ORACLE_NVFP4 ? 16 : (fmt == ORACLE_FP4G32 ? 32 : 64); }
static int fmt_scale_bytes(int fmt) { return fmt == ORACLE_INT4 ? 2 : 1; }

/* ------------------------------------------------------------------------- */
/* bf16: the upper half of an IEEE binary32.                                 */
/* ------------------------------------------------------------------------- */

float oracle_bf16_decode(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* Nearest bf16 to a finite double, ties to the even significand.  The two
 * candidates are the bf16 grid points on either side of |x| (8 significant
 * bits; fixed spacing 2^-133 below the normal range). */
uint16_t oracle_bf16_round(double x) {
    uint16_t sign = signbit(x) ? 0x8000u : 0u;
    double a = fabs(x);
    if (a == 0.0) return sign;
    int e;
    frexp(a, &e);                 /* a = f * 2^e, f in [0.5, 1) */
    int q = e - 8;                /* spacing of an 8-bit significand */
    if (q < -133) q = -133;
    double ulp = ldexp(1.0, q);
    double lo = floor(a / ulp) * ulp;
    double hi = lo + ulp;
    double r;
    if (a - lo < hi - a) {
        r = lo;
    } else if (hi - a < a - lo) {
        r = hi;
    } else {
        double n = lo / ulp;      /* integer significand of lo */
        r = (fmod(n, 2.0) == 0.0) ? lo : hi;
    }
    float rf = (float)r;          /* exact: r has at most 8 significant bits */
    uint32_t u;
    memcpy(&u, &rf, sizeof u);
    return (uint16_t)((u >> 16) | sign);
}

/* ------------------------------------------------------------------------- */
/* FP4 E2M1: sign, 2 exponent bits (bias 1), 1 mantissa bit, no inf/NaN.     */
/* ------------------------------------------------------------------------- */

float oracle_e2m1_decode(uint8_t code) {
    int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
    float mag = (e == 0) ? 0.5f * (float)m : ldexpf(1.0f + 0.5f * (float)m, e - 1);
    return s ? -mag : mag;
}

/* Nearest of the 8 non-negative E2M1 magnitudes to |v| (ties: even code),
 * which also saturates at 6; the sign bit is the sign of v. */
uint8_t oracle_e2m1_round(float v) {
    float a = fabsf(v);
    int best = 0;
    double bestd = INFINITY;
    for (int c = 0; c < 8; ++c) {
        double d = fabs((double)oracle_e2m1_decode((uint8_t)c) - (double)a);
        if (d < bestd || (d == bestd && (c & 1) == 0)) {
            best = c;
            bestd = d;
        }
    }
    return (uint8_t)(best | (signbit(v) ? 8 : 0));
}

/* ------------------------------------------------------------------------- */
/* FP8 E4M3 (finite-only variant): 4 exponent bits (bias 7), 3 mantissa bits,*/
/* S.1111.111 is NaN, largest finite 448.  Scales are non-negative.          */
/* ------------------------------------------------------------------------- */

float oracle_e4m3_decode(uint8_t code) {
    int s = (code >> 7) & 1, e = (code >> 3) & 15, m = code & 7;
    if (e == 15 && m == 7) return NAN;
    float mag = (e == 0) ? ldexpf((float)m / 8.0f, -6) : ldexpf(1.0f + (float)m / 8.0f, e - 7);
    return s ? -mag : mag;
}

/* Nearest non-negative finite E4M3 value (codes 0x00..0x7E), ties to the even
 * code; anything above 448 saturates to 448. */
uint8_t oracle_e4m3_round_sat(float s) {
    int best = 0;
    double bestd = INFINITY;
    for (int c = 0; c <= 0x7E; ++c) {
        double d = fabs((double)oracle_e4m3_decode((uint8_t)c) - (double)s);
        if (d < bestd || (d == bestd && (c & 1) == 0)) {
            best = c;
            bestd = d;
        }
    }
    return (uint8_t)best;
}

/* ------------------------------------------------------------------------- */
/* IEEE binary16: 5 exponent bits (bias 15), 10 mantissa bits.               */
/* ------------------------------------------------------------------------- */

float oracle_fp16_decode(uint16_t h) {
    int s = (h >> 15) & 1, e = (h >> 10) & 31, m = h & 1023;
    float mag;
    if (e == 31) mag = m ? NAN : INFINITY;
    else if (e == 0) mag = ldexpf((float)m, -24);
    else mag = ldexpf(1.0f + (float)m / 1024.0f, e - 15);
    return s ? -mag : mag;
}

/* Nearest non-negative finite fp16 value (codes 0x0000..0x7BFF are increasing
 * in value; binary search for the bracketing pair), ties to the even code;
 * saturates at 65504. */
uint16_t oracle_fp16_round_sat(float s) {
    double a = (double)s;
    if (a <= 0.0) return 0;
    int lo = 0, hi = 0x7BFF;
    if (a >= (double)oracle_fp16_decode((uint16_t)hi)) return (uint16_t)hi;
    while (hi - lo > 1) {           /* invariant: value(lo) <= a < value(hi) */
        int mid = (lo + hi) / 2;
        if ((double)oracle_fp16_decode((uint16_t)mid) <= a) lo = mid; else hi = mid;
    }
    double dl = a - (double)oracle_fp16_decode((uint16_t)lo);
    double dh = (double)oracle_fp16_decode((uint16_t)hi) - a;
    if (dl < dh) return (uint16_t)lo;
    if (dh < dl) return (uint16_t)hi;
    return (uint16_t)((lo & 1) == 0 ? lo : hi);
}

/* Round half to even to an integer (exact for |x| < 2^23). */
static float round_half_even(float x) {
    float f = floorf(x);
    float d = x - f;
    if (d > 0.5f) return f + 1.0f;
    if (d < 0.5f) return f;
    return (fmodf(f, 2.0f) == 0.0f) ? f : f + 1.0f;
}

/* ------------------------------------------------------------------------- */
/* Group quantizers (Sec. 3 quantizer, groups of Sec. 5.1).                  */
/* Codes come out one per byte (low nibble); callers pack.                   */
/* ------------------------------------------------------------------------- */

/* FP4: g values -> g E2M1 codes + one E4M3 scale (g = 16 NVFP4, 32 FP4 g32). */
static void quant_group_fp4(int g, const float *v, uint8_t *codes, uint8_t *scale) {
    float amax = 0.0f;
    for (int i = 0; i < g; ++i) amax = fmaxf(amax, fabsf(v[i]));
    float s32 = amax / 6.0f;                       /* q_max = 6 for E2M1 */
    uint8_t s8 = oracle_e4m3_round_sat(s32);
    float sd = oracle_e4m3_decode(s8);
    *scale = s8;
    if (sd == 0.0f) {
        for (int i = 0; i < g; ++i) codes[i] = 0;
        return;
    }
    float inv = 1.0f / sd;
    for (int i = 0; i < g; ++i) codes[i] = oracle_e2m1_round(v[i] * inv);
}

void oracle_quant_group_nvfp4(const float *v, uint8_t *codes, uint8_t *scale) {
    quant_group_fp4(16, v, codes, scale);
}

void oracle_quant_group_fp4g32(const float *v, uint8_t *codes, uint8_t *scale) {
    quant_group_fp4(32, v, codes, scale);
}

/* INT4: 64 values -> 64 signed codes in [-7, 7] (4-bit two's complement in the
 * low nibble) + one fp16 scale. */
void oracle_quant_group_int4(const float *v, uint8_t *codes, uint16_t *scale) {
    float amax = 0.0f;
    for (int i = 0; i < 64; ++i) amax = fmaxf(amax, fabsf(v[i]));
    float s32 = amax / 7.0f;                       /* q_max = 2^(4-1) - 1 */
    uint16_t sh = oracle_fp16_round_sat(s32);
    float sd = oracle_fp16_decode(sh);
    *scale = sh;
    if (sd == 0.0f) {
        for (int i = 0; i < 64; ++i) codes[i] = 0;
        return;
    }
    float inv = 1.0f / sd;
    for (int i = 0; i < 64; ++i) {
        float q = round_half_even(v[i] * inv);
        if (q > 7.0f) q = 7.0f;
        if (q < -7.0f) q = -7.0f;
        codes[i] = (uint8_t)((int)q & 0xF);
    }
}

static float deq_code(int fmt, uint8_t code) {
    if (fmt != ORACLE_INT4) return oracle_e2m1_decode(code & 0xF);
    int q = code & 0xF;
    return (float)(q >= 8 ? q - 16 : q);
}

static uint8_t get_nibble(const uint8_t *packed, long i) {
    uint8_t b = packed[i >> 1];
    return (i & 1) ? (uint8_t)(b >> 4) : (uint8_t)(b & 0xF);
}

static void quantize_row(int fmt, const float *v, int K, uint8_t *codes_row, void *scales_row) {
    int g = fmt_group(fmt);
    uint8_t c[64];
    for (int k0 = 0; k0 < K; k0 += g) {
        if (fmt != ORACLE_INT4)
            quant_group_fp4(g, v + k0, c, (uint8_t *)scales_row + k0 / g);
        else
            oracle_quant_group_int4(v + k0, c, (uint16_t *)scales_row + k0 / g);
        for (int i = 0; i < g; i += 2)
            codes_row[(k0 + i) / 2] = (uint8_t)((c[i] & 0xF) | ((c[i + 1] & 0xF) << 4));
    }
}

/* ------------------------------------------------------------------------- */
/* Activation side (the fused "quantize + down-projection" of Sec. 4.3; the  */
/* smoothing X_hat = X diag(lambda)^-1 and the branch X_hat L1 of Sec. 4.2). */
/*   x_hat[m,k] = fp32(x[m,k]) * inv_lambda[k]        (one fp32 rounding)     */
/*   codes/scales = Q(x_hat) per group                                         */
/*   XL1[m,j]   = sum_k x_hat[m,k] * L1[k,j], fp32 products and sums in       */
/*                increasing k (kept fp32)                                     */
/* X: M x K bf16; L1: K x r bf16 (row-major); codes: M x K/2 bytes (element  */
/* 2i in the low nibble); scales: M x K/g (uint8 E4M3 or uint16 fp16); XL1:   */
/* M x r fp32.  inv_lambda may be NULL (lambda = 1).                           */
/* ------------------------------------------------------------------------- */
int oracle_act_quant(int fmt, int M, int K, int r, const uint16_t *X, const float *inv_lambda,
                     const uint16_t *L1, uint8_t *codes, void *scales, float *XL1) {
    int g = fmt_group(fmt);
    if (K % g) return 1;
    int ssz = fmt_scale_bytes(fmt);
#pragma omp parallel
    {
        float *xh = (float *)__builtin_alloca(sizeof(float) * (size_t)K);
        float *xf = (float *)__builtin_alloca(sizeof(float) * (size_t)K);
#pragma omp for schedule(static)
        for (int m = 0; m < M; ++m) {
            const uint16_t *xr = X + (long)m * K;
            for (int k = 0; k < K; ++k) {
                xf[k] = oracle_bf16_decode(xr[k]);
                xh[k] = inv_lambda ? xf[k] * inv_lambda[k] : xf[k];
            }
            quantize_row(fmt, xh, K, codes + (long)m * (K / 2),
                         (uint8_t *)scales + (long)m * (K / g) * ssz);
            for (int j = 0; j < r; ++j) {
                float acc = 0.0f;
                for (int k = 0; k < K; ++k)
                    acc += xh[k] * oracle_bf16_decode(L1[(long)k * r + j]);
                XL1[(long)m * r + j] = acc;
            }
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------- */
/* Weight side: quantize the residual R (K x N fp32, row-major) along K for  */
/* each output column n.  codes: N x K/2, scales: N x K/g.                    */
/* ------------------------------------------------------------------------- */
int oracle_weight_quant(int fmt, int K, int N, const float *R, uint8_t *codes, void *scales) {
    int g = fmt_group(fmt);
    if (K % g) return 1;
    int ssz = fmt_scale_bytes(fmt);
#pragma omp parallel
    {
        float *col = (float *)__builtin_alloca(sizeof(float) * (size_t)K);
#pragma omp for schedule(static)
        for (int n = 0; n < N; ++n) {
            for (int k = 0; k < K; ++k) col[k] = R[(long)k * N + n];
            quantize_row(fmt, col, K, codes + (long)n * (K / 2),
                         (uint8_t *)scales + (long)n * (K / g) * ssz);
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------- */
/* The layer output (Eq. 5 of Sec. 4.2 plus bias):                            */
/*   y[m,n] = bf16( sum_g s_x[m,g] s_w[n,g] sum_{k in g} deq(qx) deq(qw)      */
/*                  + sum_j XL1[m,j] L2[j,n] + bias[n] )   (XL1 fp32)         */
/* for the rows listed in `rows` (all rows if rows == NULL, n_rows = M) and   */
/* all N columns; Y is n_rows x N bf16.  L2: r x N bf16; bias may be NULL.   */
/* ------------------------------------------------------------------------- */
/* w_exp: the weight codes and scales are those of R * 2^w_exp (the optional
 * power-of-two prescale of the weight residual); the group sum is multiplied
 * by 2^-w_exp (exact) before the branch and the bias are added. */
int oracle_linear_rows(int fmt, int M, int N, int K, int r, const uint8_t *codes_x,
                       const void *scales_x, const float *XL1, const uint8_t *codes_w,
                       const void *scales_w, const uint16_t *L2, const uint16_t *bias,
                       const int *rows, int n_rows, int w_exp, uint16_t *Y) {
    int g = fmt_group(fmt);
    if (K % g) return 1;
    int G = K / g;
#pragma omp parallel for schedule(dynamic, 1)
    for (int i = 0; i < n_rows; ++i) {
        int m = rows ? rows[i] : i;
        if (m < 0 || m >= M) continue;
        const uint8_t *cx = codes_x + (long)m * (K / 2);
        for (int n = 0; n < N; ++n) {
            const uint8_t *cw = codes_w + (long)n * (K / 2);
            float acc = 0.0f;
            for (int gi = 0; gi < G; ++gi) {
                float sx, sw;
                if (fmt != ORACLE_INT4) {
                    sx = oracle_e4m3_decode(((const uint8_t *)scales_x)[(long)m * G + gi]);
                    sw = oracle_e4m3_decode(((const uint8_t *)scales_w)[(long)n * G + gi]);
                } else {
                    sx = oracle_fp16_decode(((const uint16_t *)scales_x)[(long)m * G + gi]);
                    sw = oracle_fp16_decode(((const uint16_t *)scales_w)[(long)n * G + gi]);
                }
                float part = 0.0f;  /* exact: multiples of 1/4 below 2^12, or integers below 2^12 */
                for (int k = gi * g; k < (gi + 1) * g; ++k)
                    part += deq_code(fmt, get_nibble(cx, k)) * deq_code(fmt, get_nibble(cw, k));
                acc += (sx * sw) * part;
            }
            acc = ldexpf(acc, -w_exp);
            for (int j = 0; j < r; ++j)
                acc += XL1[(long)m * r + j] * oracle_bf16_decode(L2[(long)j * N + n]);
            if (bias) acc += oracle_bf16_decode(bias[n]);
            Y[(long)i * N + n] = oracle_bf16_round((double)acc);
        }
    }
    return 0;
}

/* Dequantize packed codes + scales (rows x K) to fp32: s * deq(q). */
int oracle_dequant(int fmt, int rows, int K, const uint8_t *codes, const void *scales, float *out) {
    int g = fmt_group(fmt);
    if (K % g) return 1;
    int G = K / g;
    for (long i = 0; i < rows; ++i)
        for (int k = 0; k < K; ++k) {
            float s = (fmt != ORACLE_INT4)
                          ? oracle_e4m3_decode(((const uint8_t *)scales)[i * G + k / g])
                          : oracle_fp16_decode(((const uint16_t *)scales)[i * G + k / g]);
            out[i * K + k] = s * deq_code(fmt, get_nibble(codes + i * (K / 2), k));
        }
    return 0;
}

/* Element-wise helpers for the Python side of the oracle. */
void oracle_bf16_round_array(const double *x, long n, uint16_t *out) {
    for (long i = 0; i < n; ++i) out[i] = oracle_bf16_round(x[i]);
}

void oracle_e4m3_round_array(const float *x, long n, uint8_t *out) {
    for (long i = 0; i < n; ++i) out[i] = oracle_e4m3_round_sat(x[i]);
}

void oracle_e2m1_round_array(const float *x, long n, uint8_t *out) {
    for (long i = 0; i < n; ++i) out[i] = oracle_e2m1_round(x[i]);
}

void oracle_fp16_round_array(const float *x, long n, uint16_t *out) {
    for (long i = 0; i < n; ++i) out[i] = oracle_fp16_round_sat(x[i]);
}

/* ------------------------------------------------------------------------- */
/* W8A8 (Sec. 5.1 "Implementation details", 8-bit setting): per-token dynamic */
/* activation quantization and per-channel weight quantization, q_max = 127   */
/* (Sec. 3: 2^(b-1) - 1 for signed b-bit integers).                           */
/*   s = amax / 127 (IEEE fp32, kept in fp32: a dynamic scale has no storage  */
/*   format of its own); q = clamp(rint_even(v * RN(1/s)), -127, 127); s = 0  */
/*   gives zero codes.                                                         */
/* ------------------------------------------------------------------------- */
static void quant_int8(const float *v, long n, long stride, int8_t *codes, float *scale) {
    float amax = 0.0f;
    for (long i = 0; i < n; ++i) amax = fmaxf(amax, fabsf(v[i * stride]));
    float s = amax / 127.0f;
    *scale = s;
    if (s == 0.0f) {
        for (long i = 0; i < n; ++i) codes[i] = 0;
        return;
    }
    float inv = 1.0f / s;
    for (long i = 0; i < n; ++i) {
        float q = round_half_even(v[i * stride] * inv);
        if (q > 127.0f) q = 127.0f;
        if (q < -127.0f) q = -127.0f;
        codes[i] = (int8_t)q;
    }
}

/* Activations: codes M x K int8, scales M fp32, XL1 M x r fp32 (X_hat L1 as above). */
int oracle_act_quant_w8(int M, int K, int r, const uint16_t *X, const float *inv_lambda,
                        const uint16_t *L1, int8_t *codes, float *scales, float *XL1) {
#pragma omp parallel
    {
        float *xh = (float *)__builtin_alloca(sizeof(float) * (size_t)K);
        float *xf = (float *)__builtin_alloca(sizeof(float) * (size_t)K);
#pragma omp for schedule(static)
        for (int m = 0; m < M; ++m) {
            const uint16_t *xr = X + (long)m * K;
            for (int k = 0; k < K; ++k) {
                xf[k] = oracle_bf16_decode(xr[k]);
                xh[k] = inv_lambda ? xf[k] * inv_lambda[k] : xf[k];
            }
            quant_int8(xh, K, 1, codes + (long)m * K, scales + m);
            for (int j = 0; j < r; ++j) {
                float acc = 0.0f;
                for (int k = 0; k < K; ++k)
                    acc += xh[k] * oracle_bf16_decode(L1[(long)k * r + j]);
                XL1[(long)m * r + j] = acc;
            }
        }
    }
    return 0;
}

/* Weights: R K x N fp32 -> codes N x K int8 (per output channel), scales N fp32. */
int oracle_weight_quant_w8(int K, int N, const float *R, int8_t *codes, float *scales) {
#pragma omp parallel for schedule(static)
    for (int n = 0; n < N; ++n) quant_int8(R + n, K, N, codes + (long)n * K, scales + n);
    return 0;
}

/* y[m,n] = bf16( float(sum_k qx qw) * (s_x[m] s_w[n]) + sum_j XL1[m,j] L2[j,n] + bias[n] ):
 * the integer dot product is exact (|sum| < 127^2 K < 2^31 for K < 2^17) and
 * rounded once to fp32. */
int oracle_linear_rows_w8(int M, int N, int K, int r, const int8_t *codes_x, const float *scales_x,
                          const float *XL1, const int8_t *codes_w, const float *scales_w,
                          const uint16_t *L2, const uint16_t *bias, const int *rows, int n_rows,
                          uint16_t *Y) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int i = 0; i < n_rows; ++i) {
        int m = rows ? rows[i] : i;
        if (m < 0 || m >= M) continue;
        const int8_t *cx = codes_x + (long)m * K;
        for (int n = 0; n < N; ++n) {
            const int8_t *cw = codes_w + (long)n * K;
            long long dot = 0;
            for (int k = 0; k < K; ++k) dot += (long long)cx[k] * (long long)cw[k];
            float acc = (float)dot * (scales_x[m] * scales_w[n]);
            for (int j = 0; j < r; ++j)
                acc += XL1[(long)m * r + j] * oracle_bf16_decode(L2[(long)j * N + n]);
            if (bias) acc += oracle_bf16_decode(bias[n]);
            Y[(long)i * N + n] = oracle_bf16_round((double)acc);
        }
    }
    return 0;
}
