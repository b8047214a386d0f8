/*
 * cider_oracle.c -- plain, slow CPU oracle for the W8A8 / W4A8
 * activation-quantized linear.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or
 * load this file: only the tests, the smoke check and the benchmark's CPU
 * baseline leg use it.  It shares no code, header, table or helper with the
 * CUDA library; it is compiled with gcc -O2 -ffp-contract=off (no fast-math),
 * so every float operation below is one IEEE-754 operation, rounded once.
 *
 * Sources (page title, then section):
 *  [BLOG]   juejin post "在Mac上跑大模型，MLX 不是终点",
 *           section "W8A8 对称量化：Cider 的选择" (per-token scale = max|x|/127,
 *           x_int8 = round(x/scale) clamped to [-128,127], y = (x_int8 . w_int8)
 *           * scale_x * scale_w), section "INT8 TensorOps 内核设计" (INT32
 *           accumulator, dequant fused in the store), section "三种量化粒度的实现"
 *           (per-channel vs per-group gs=128/64 weight scales; per-group
 *           dequant is a piecewise multiply).
 *  [README] Cider README (WeHub community translation), table "量化"
 *           (weights symmetric INT8 per-channel or per-group gs=64/128;
 *           W4A8 weights symmetric INT4 "zp=8"; activations symmetric INT8
 *           per-token; INT32 accumulation; C_fp16 = C_int32 * s_act * s_weight),
 *           table "模式" (W4A8: INT4 packed in uint8, unpack -> TensorOps),
 *           section "底层 API" (quantize_weight_int8, pack_weight_int4),
 *           section "Metal Kernel 流水线" (Decode: INT8 matrix-vector
 *           product, weights dequantized on the fly, no activation
 *           quantization).
 *
 * Readings where the pages are silent (each one is listed in the design notes):
 *  - round() is round-half-away-from-zero;
 *  - scale_x, scale_w are fp32; t = x / scale_x is one correctly rounded fp32
 *    division by the stored scale (not a multiply by 127/amax);
 *  - an all-zero token has scale 0 and q = 0;
 *  - clip_percentile: the percentile of the magnitudes |w| of a slab, by
 *    linear interpolation at position p/100*(len-1) (the t of that position
 *    rounded once to fp32, the interpolation in fp32), codes clipped to
 *    [-127, 127]; a zero percentile falls back to max|w|;
 *  - INT4 weights: q in [-8,7] from scale = max|w_group|/7, stored as the
 *    offset-binary nibble q+8, two per byte, low nibble = even k;
 *  - the dequant is evaluated in fp64 here and rounded once to fp16/bf16
 *    (round to nearest even); the per-group sum runs over groups in
 *    ascending order.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_F16 0
#define ORACLE_BF16 1

/* ---------------------------------------------------------------------- */
/* Number formats, from the IEEE 754 definitions.                          */
/* ---------------------------------------------------------------------- */

/* binary16: 1 sign, 5 exponent (bias 15), 10 fraction bits. */
float oracle_f16_to_f32(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int f = h & 0x3ff;
    double v;
    if (e == 0x1f) {
        v = f ? NAN : INFINITY;
    } else if (e == 0) {
        v = ldexp((double)f, -24); /* subnormal: f * 2^(1-15-10) */
    } else {
        v = ldexp((double)(f + 1024), e - 25); /* (1024+f) * 2^(e-15-10) */
    }
    return (float)(sign ? -v : v); /* exact: binary16 is a subset of binary32 */
}

/* bfloat16: the upper 16 bits of a binary32. */
float oracle_bf16_to_f32(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* Round a double to the nearest value of a binary format with `mant` stored
 * fraction bits and `ebits` exponent bits, ties to even; overflow goes to
 * +-inf.  Returns the format's bit pattern. */
static uint32_t round_to_format(double v, int mant, int ebits)
{
    const int bias = (1 << (ebits - 1)) - 1;
    const int emin = 1 - bias;
    const uint32_t sign = signbit(v) ? 1u : 0u;
    const uint32_t sign_bit = sign << (mant + ebits);
    const uint32_t exp_all_ones = ((1u << ebits) - 1u) << mant;
    if (isnan(v))
        return sign_bit | exp_all_ones | (1u << (mant - 1));
    double a = fabs(v);
    if (isinf(a))
        return sign_bit | exp_all_ones;
    if (a == 0.0)
        return sign_bit;
    int ex;
    (void)frexp(a, &ex); /* a = fr * 2^ex, fr in [0.5, 1) */
    int E = ex - 1;      /* 2^E <= a < 2^(E+1) */
    if (E < emin)
        E = emin; /* subnormal range: fixed quantum */
    double scaled = ldexp(a, mant - E); /* a / quantum, exact */
    double fl = floor(scaled);
    double diff = scaled - fl; /* exact: scaled < 2^(mant+1) + 1 */
    double r = fl;
    if (diff > 0.5 || (diff == 0.5 && fmod(fl, 2.0) != 0.0))
        r = fl + 1.0;
    if (r >= ldexp(1.0, mant + 1)) { /* carried into the next binade */
        r = ldexp(1.0, mant);
        E += 1;
    }
    if (E > bias)
        return sign_bit | exp_all_ones; /* overflow */
    uint32_t ri = (uint32_t)r;
    if (ri < (1u << mant)) /* subnormal (E == emin) */
        return sign_bit | ri;
    return sign_bit | ((uint32_t)(E + bias) << mant) | (ri - (1u << mant));
}

uint16_t oracle_f64_to_f16_rne(double v) { return (uint16_t)round_to_format(v, 10, 5); }
uint16_t oracle_f64_to_bf16_rne(double v) { return (uint16_t)round_to_format(v, 7, 8); }

static float widen(const uint16_t* x, int64_t i, int dt)
{
    return dt == ORACLE_BF16 ? oracle_bf16_to_f32(x[i]) : oracle_f16_to_f32(x[i]);
}

static uint16_t narrow(double v, int dt)
{
    return dt == ORACLE_BF16 ? oracle_f64_to_bf16_rne(v) : oracle_f64_to_f16_rne(v);
}

/* round(t), halfway cases away from zero.  t - trunc(t) is exact in fp32. */
float oracle_round_half_away(float t)
{
    float r = truncf(t);
    float d = t - r;
    if (fabsf(d) >= 0.5f)
        r += (t > 0.0f) ? 1.0f : -1.0f;
    return r;
}

static int clamp_int(float r, int lo, int hi)
{
    if (r < (float)lo)
        return lo;
    if (r > (float)hi)
        return hi;
    return (int)r;
}

/* ---------------------------------------------------------------------- */
/* Online per-token activation quantization  [BLOG "W8A8 对称量化"]        */
/*   scale = max|x| / 127 ;  q = clamp(round(x / scale), -128, 127)       */
/* ---------------------------------------------------------------------- */
void oracle_quantize_act(const uint16_t* x, int xdt, int64_t M, int64_t K,
                         int8_t* q, float* sx)
{
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        float amax = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            float a = fabsf(widen(x, m * K + k, xdt));
            if (a > amax)
                amax = a;
        }
        float s = amax / 127.0f;
        sx[m] = s;
        for (int64_t k = 0; k < K; ++k) {
            if (amax == 0.0f) {
                q[m * K + k] = 0;
                continue;
            }
            float t = widen(x, m * K + k, xdt) / s;
            q[m * K + k] = (int8_t)clamp_int(oracle_round_half_away(t), -128, 127);
        }
    }
}

/* ---------------------------------------------------------------------- */
/* Offline weight quantization  [README "底层 API" quantize_weight_int8,   */
/* pack_weight_int4; table "量化"; BLOG "三种量化粒度的实现"]               */
/* W is [N][K] (output channel n, input channel k), fp32.                  */
/* ---------------------------------------------------------------------- */

/* One symmetric scale per slab W[n, k0:k0+len]; q in [-qmax-1, qmax]. */
static void quantize_slab(const float* w, int64_t len, float qmax, int lo, int hi,
                          int8_t* qw, float* s_out)
{
    float amax = 0.0f;
    for (int64_t k = 0; k < len; ++k)
        if (fabsf(w[k]) > amax)
            amax = fabsf(w[k]);
    float s = amax / qmax;
    *s_out = s;
    for (int64_t k = 0; k < len; ++k)
        qw[k] = (amax == 0.0f) ? 0 : (int8_t)clamp_int(oracle_round_half_away(w[k] / s), lo, hi);
}

/* per output channel: sw[n] = max_k |W[n,k]| / 127 */
void oracle_quantize_weight_pc(const float* W, int64_t N, int64_t K, int8_t* qw, float* sw)
{
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n)
        quantize_slab(W + n * K, K, 127.0f, -128, 127, qw + n * K, sw + n);
}

/* per group of gs input channels: sw[n][g] = max |W[n, g*gs:(g+1)*gs]| / 127 */
void oracle_quantize_weight_pg(const float* W, int64_t N, int64_t K, int64_t gs,
                               int8_t* qw, float* sw)
{
    const int64_t G = K / gs;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n)
        for (int64_t g = 0; g < G; ++g)
            quantize_slab(W + n * K + g * gs, gs, 127.0f, -128, 127, qw + n * K + g * gs,
                          sw + n * G + g);
}

/* ---------------------------------------------------------------------- */
/* Percentile-clipped weight scales  [README "说明": the conversion takes   */
/* its scales by min-max by default and also supports a percentile method, */
/* clip_percentile=99.9]                                                    */
/* The clipping value c of a slab is the p-th percentile of its magnitudes */
/* |w|, linearly interpolated between order statistics (the common         */
/* definition: position p/100 * (len-1) in the ascending order); scale =   */
/* c / 127 and codes clip symmetrically to [-127, 127].  A slab whose      */
/* percentile is 0 (mostly zeros) takes c = max|w| instead.                */
/* ---------------------------------------------------------------------- */

/* Position of the p-th percentile among len ascending values: index i of
 * the lower neighbour and the fraction t towards the next one.  Evaluated
 * in double, t rounded once to float. */
void oracle_percentile_position(double p, int64_t len, int64_t* i_out, float* t_out)
{
    double pos = p / 100.0 * (double)(len - 1);
    int64_t i = (int64_t)floor(pos);
    if (i > len - 1)
        i = len - 1;
    if (i < 0)
        i = 0;
    *i_out = i;
    *t_out = (float)(pos - (double)i);
}

static int cmp_float_asc(const void* a, const void* b)
{
    float x = *(const float*)a, y = *(const float*)b;
    return (x > y) - (x < y);
}

/* p-th percentile of |w[0..len)|: sort the magnitudes, then
 * v = a[i] + t * (a[i+1] - a[i]) in three rounded fp32 operations. */
static float abs_percentile(const float* w, int64_t len, int64_t i, float t)
{
    float* a = (float*)malloc((size_t)len * sizeof(float));
    for (int64_t k = 0; k < len; ++k)
        a[k] = fabsf(w[k]);
    qsort(a, (size_t)len, sizeof(float), cmp_float_asc);
    float v = a[i];
    if (t != 0.0f && i + 1 < len) {
        float d = a[i + 1] - a[i];
        float td = t * d;
        v = a[i] + td;
    }
    free(a);
    return v;
}

static void quantize_slab_clip(const float* w, int64_t len, int64_t i, float t, int8_t* qw, float* s_out)
{
    float amax = 0.0f;
    for (int64_t k = 0; k < len; ++k)
        if (fabsf(w[k]) > amax)
            amax = fabsf(w[k]);
    float v = abs_percentile(w, len, i, t);
    float c = (v == 0.0f) ? amax : v;
    float s = c / 127.0f;
    *s_out = s;
    for (int64_t k = 0; k < len; ++k)
        qw[k] = (c == 0.0f) ? 0 : (int8_t)clamp_int(oracle_round_half_away(w[k] / s), -127, 127);
}

/* per output channel, clipped: sw[n] = pct_p(|W[n,:]|) / 127 */
void oracle_quantize_weight_pc_clip(const float* W, int64_t N, int64_t K, double p, int8_t* qw, float* sw)
{
    int64_t i;
    float t;
    oracle_percentile_position(p, K, &i, &t);
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n)
        quantize_slab_clip(W + n * K, K, i, t, qw + n * K, sw + n);
}

/* per group of gs, clipped: sw[n][g] = pct_p(|W[n, g*gs:(g+1)*gs]|) / 127 */
void oracle_quantize_weight_pg_clip(const float* W, int64_t N, int64_t K, int64_t gs, double p,
                                    int8_t* qw, float* sw)
{
    const int64_t G = K / gs;
    int64_t i;
    float t;
    oracle_percentile_position(p, gs, &i, &t);
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n)
        for (int64_t g = 0; g < G; ++g)
            quantize_slab_clip(W + n * K + g * gs, gs, i, t, qw + n * K + g * gs, sw + n * G + g);
}

/* INT4, per group: q in [-8,7] from scale max|w|/7, packed as nibble q+8,
 * byte j of row n holds k=2j in its low nibble and k=2j+1 in its high one. */
void oracle_quantize_weight_int4_pg(const float* W, int64_t N, int64_t K, int64_t gs,
                                    uint8_t* packed, float* sw)
{
    const int64_t G = K / gs;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n)
        for (int64_t g = 0; g < G; ++g) {
            const float* wg = W + n * K + g * gs;
            float amax = 0.0f;
            for (int64_t k = 0; k < gs; ++k)
                if (fabsf(wg[k]) > amax)
                    amax = fabsf(wg[k]);
            float s = amax / 7.0f;
            sw[n * G + g] = s;
            for (int64_t k = 0; k < gs; ++k) {
                int qv = (amax == 0.0f) ? 0 : clamp_int(oracle_round_half_away(wg[k] / s), -8, 7);
                int64_t kk = g * gs + k;
                uint8_t nib = (uint8_t)(qv + 8);
                uint8_t* b = &packed[n * (K / 2) + kk / 2];
                if ((kk & 1) == 0)
                    *b = (uint8_t)((*b & 0xF0) | nib);
                else
                    *b = (uint8_t)((*b & 0x0F) | (nib << 4));
            }
        }
}

/* [README table "模式": INT4 packed (uint8), unpack -> INT8] */
void oracle_unpack_int4(const uint8_t* packed, int64_t N, int64_t K, int8_t* w)
{
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) {
            uint8_t b = packed[n * (K / 2) + k / 2];
            int nib = (k & 1) ? (b >> 4) : (b & 0x0F);
            w[n * K + k] = (int8_t)(nib - 8);
        }
}

/* ---------------------------------------------------------------------- */
/* INT8 x INT8 -> INT32 GEMM  [BLOG "INT8 TensorOps 内核设计"]             */
/* acc[m][n] = sum_k q[m][k] * w[n][k]; summed in int64, must fit int32.   */
/* Returns 0, or -1 if any sum leaves the int32 range.                     */
/* ---------------------------------------------------------------------- */
int oracle_gemm_i32(const int8_t* q, const int8_t* w, int64_t M, int64_t N, int64_t K,
                    int32_t* acc)
{
    int bad = 0;
#pragma omp parallel for schedule(static) reduction(| : bad)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            int64_t s = 0;
            for (int64_t k = 0; k < K; ++k)
                s += (int64_t)q[m * K + k] * (int64_t)w[n * K + k];
            if (s > INT32_MAX || s < INT32_MIN)
                bad = 1;
            acc[m * N + n] = (int32_t)s;
        }
    return bad ? -1 : 0;
}

/* Per-group partial sums: acc_g[g][m][n] = sum_{k in group g} q[m][k]*w[n][k]. */
int oracle_gemm_i32_grouped(const int8_t* q, const int8_t* w, int64_t M, int64_t N,
                            int64_t K, int64_t gs, int32_t* acc_g)
{
    const int64_t G = K / gs;
    int bad = 0;
#pragma omp parallel for schedule(static) reduction(| : bad)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n)
            for (int64_t g = 0; g < G; ++g) {
                int64_t s = 0;
                for (int64_t k = g * gs; k < (g + 1) * gs; ++k)
                    s += (int64_t)q[m * K + k] * (int64_t)w[n * K + k];
                if (s > INT32_MAX || s < INT32_MIN)
                    bad = 1;
                acc_g[(g * M + m) * N + n] = (int32_t)s;
            }
    return bad ? -1 : 0;
}

/* ---------------------------------------------------------------------- */
/* Dequant  [README table "量化": C_fp16 = C_int32 * s_act * s_weight]     */
/* ---------------------------------------------------------------------- */
void oracle_dequant_pc(const int32_t* acc, const float* sx, const float* sw, int64_t M,
                       int64_t N, int ydt, uint16_t* y)
{
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n)
            y[m * N + n] = narrow((double)acc[m * N + n] * (double)sx[m] * (double)sw[n], ydt);
}

/* per-group: y = scale_x * sum_g acc_g * scale_w[n][g]  [BLOG "三种量化粒度的实现"] */
void oracle_dequant_pg(const int32_t* acc_g, const float* sx, const float* sw, int64_t M,
                       int64_t N, int64_t G, int ydt, uint16_t* y)
{
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double s = 0.0;
            for (int64_t g = 0; g < G; ++g)
                s += (double)acc_g[(g * M + m) * N + n] * (double)sw[n * G + g];
            y[m * N + n] = narrow((double)sx[m] * s, ydt);
        }
}

/* ---------------------------------------------------------------------- */
/* Whole linears, row by row (rows are independent, so any subset of rows  */
/* of x gives exactly those rows of y).                                    */
/* ---------------------------------------------------------------------- */

/* W8A8, per-channel weight scales. */
int oracle_linear_pc(const uint16_t* x, int xdt, int64_t M, int64_t K, const int8_t* w,
                     const float* sw, int64_t N, int ydt, uint16_t* y)
{
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int64_t m = 0; m < M; ++m) {
        int8_t qrow[K > 0 ? K : 1];
        float s;
        oracle_quantize_act(x + m * K, xdt, 1, K, qrow, &s);
        for (int64_t n = 0; n < N; ++n) {
            int64_t a = 0;
            for (int64_t k = 0; k < K; ++k)
                a += (int64_t)qrow[k] * (int64_t)w[n * K + k];
            if (a > INT32_MAX || a < INT32_MIN)
                bad = 1;
            y[m * N + n] = narrow((double)(int32_t)a * (double)s * (double)sw[n], ydt);
        }
    }
    return bad ? -1 : 0;
}

/* W8A16 decode product, per-channel weight scales ([README] section
 * "Metal Kernel 流水线", Decode: a direct INT8 matrix-vector product with the
 * weights dequantized on the fly and no activation quantization):
 * y[m,n] = round(sw[n] * sum_k x[m,k] * w[n,k]) -- x widened exactly, the
 * products and their sum in fp64, one rounding to the output type. */
int oracle_w8a16_linear_pc(const uint16_t* x, int xdt, int64_t M, int64_t K, const int8_t* w,
                           const float* sw, int64_t N, int ydt, uint16_t* y)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            double a = 0.0;
            for (int64_t k = 0; k < K; ++k)
                a += (double)widen(x, m * K + k, xdt) * (double)w[n * K + k];
            y[m * N + n] = narrow(a * (double)sw[n], ydt);
        }
    }
    return 0;
}

/* W8A16 decode product, per-group weight scales sw[n][K/gs] ([README]
 * section "Metal Kernel 流水线", Decode, and the per-group INT8 MV kernel of the
 * project's kernel list): the weights of group g of row n are dequantized by
 * sw[n][g] on the fly, the activations are used as they are:
 * y[m,n] = round(sum_g sw[n][g] * sum_{k in g} x[m,k] * w[n,k]), x widened
 * exactly, each group's sum and the sum over groups (ascending g) in fp64,
 * one rounding to the output type. */
int oracle_w8a16_linear_pg(const uint16_t* x, int xdt, int64_t M, int64_t K, const int8_t* w,
                           const float* sw, int64_t N, int64_t gs, int ydt, uint16_t* y)
{
    const int64_t G = K / gs;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            double sum = 0.0;
            for (int64_t g = 0; g < G; ++g) {
                double part = 0.0;
                for (int64_t k = g * gs; k < (g + 1) * gs; ++k)
                    part += (double)widen(x, m * K + k, xdt) * (double)w[n * K + k];
                sum += (double)sw[n * G + g] * part;
            }
            y[m * N + n] = narrow(sum, ydt);
        }
    }
    return 0;
}

/* W8A8, per-group weight scales sw[n][K/gs]. */
int oracle_linear_pg(const uint16_t* x, int xdt, int64_t M, int64_t K, const int8_t* w,
                     const float* sw, int64_t N, int64_t gs, int ydt, uint16_t* y)
{
    const int64_t G = K / gs;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int64_t m = 0; m < M; ++m) {
        int8_t qrow[K > 0 ? K : 1];
        float s;
        oracle_quantize_act(x + m * K, xdt, 1, K, qrow, &s);
        for (int64_t n = 0; n < N; ++n) {
            double sum = 0.0;
            for (int64_t g = 0; g < G; ++g) {
                int64_t a = 0;
                for (int64_t k = g * gs; k < (g + 1) * gs; ++k)
                    a += (int64_t)qrow[k] * (int64_t)w[n * K + k];
                if (a > INT32_MAX || a < INT32_MIN)
                    bad = 1;
                sum += (double)a * (double)sw[n * G + g];
            }
            y[m * N + n] = narrow((double)s * sum, ydt);
        }
    }
    return bad ? -1 : 0;
}

/* W4A8, per-group: unpack the nibbles, then the per-group linear. */
int oracle_w4a8_linear_pg(const uint16_t* x, int xdt, int64_t M, int64_t K,
                          const uint8_t* packed, const float* sw, int64_t N, int64_t gs,
                          int ydt, uint16_t* y, int8_t* w_scratch /* [N][K] */)
{
    oracle_unpack_int4(packed, N, K, w_scratch);
    return oracle_linear_pg(x, xdt, M, K, w_scratch, sw, N, gs, ydt, y);
}

/* ---------------------------------------------------------------------- */
/* SiLU(gate) * up between the MLP linears of a decoder layer, rounded to  */
/* the activation dtype: a = round(silu(g) * u), silu(g) = g / (1 + e^-g). */
/* ---------------------------------------------------------------------- */
void oracle_silu_mul(const uint16_t* g, const uint16_t* u, int dt, int64_t n, uint16_t* a)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        double gv = (double)widen(g, i, dt);
        double uv = (double)widen(u, i, dt);
        a[i] = narrow(gv / (1.0 + exp(-gv)) * uv, dt);
    }
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ---------------------------------------------------------------------- */
/* Array forms of the scalar helpers, so the tests can sweep whole ranges. */
/* ---------------------------------------------------------------------- */
void oracle_widen_array(const uint16_t* x, int dt, int64_t n, float* out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = widen(x, i, dt);
}

void oracle_narrow_array(const double* v, int dt, int64_t n, uint16_t* out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = narrow(v[i], dt);
}

void oracle_round_half_away_array(const float* t, int64_t n, float* out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = oracle_round_half_away(t[i]);
}
