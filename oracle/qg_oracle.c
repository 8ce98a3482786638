/*
 * qg_oracle.c -- plain CPU oracle for the quantized linear layer.
 *
 * TEST INFRASTRUCTURE.  Only the tests, the smoke check and the bench's
 * cpu_baseline / reference leg may load this library.  The product path
 * (the CUDA library and its Python binding) never calls it, and the two
 * share no source: no headers, no helpers, no constants.
 *
 * Every function below is the plain definition of one step, written from the
 * pages, in this order:
 *
 *   affine quantization   x_int = round(x/s) + z ;  x_hat = (x_int - z) * s
 *       "AI Infra guide, ch.4 Quantization", sec. 1.1 (the quantization math)
 *   symmetric scale       s = max|x| / 127, z = 0            (same page, sec. 1.2 table)
 *   asymmetric scale      s = (max - min) / 255, z adjusted  (same page, sec. 1.2 table)
 *   granularity           per-channel / per-group / per-token (same page, sec. 1.3)
 *   group-wise INT4, g=128, independent scale + zero per group
 *       "LLM inference cost: W8A8/W4A8 ...", sec. 2.2 (first technique)
 *   SmoothQuant           Y = (X diag(s)^-1)(diag(s) W),
 *                         s_j = max|X_j|^a / max|W_j|^(1-a), a = 0.5
 *       "AI Infra guide, ch.4 Quantization", sec. 2.2
 *   weight-only INT4      Y = X * dequant(W)     (same page, sec. 3.1)
 *   W4A8                  4-bit weights, 8-bit activations, group-wise
 *       "LLM inference cost: W8A8/W4A8 ...", sec. 2.2
 *
 * Readings where the pages are silent, each taken as stated here:
 *   A  the asymmetric range is widened to include 0: mn' = min(min V, 0),
 *      mx' = max(max V, 0), so that z lies in [0,15] and 0 is exact;
 *   B  the 4-bit asymmetric scale divides by 15 = 2^4 - 1 (the page's 255 is 2^8 - 1);
 *   C  the fp16 scale is rounded toward +infinity, so that s >= r/15 and every
 *      element keeps the |x - x_hat| <= s/2 bound;
 *   D  the code is round(x/s) + z in that literal order, ties to even;
 *   E  8 codes per uint32 along K, low nibble first: packed[kb][n] holds
 *      k = 8kb .. 8kb+7 of column n;
 *   F  the W4A16 output dtype equals the activation dtype;
 *   G  the smoothing statistics come from a separate calibration batch;
 *   H  X~ = X * inv_s with inv_s = 1/s formed first (one fp32 rounding each);
 *      W~ = W * s (one fp32 rounding);
 *   I  symmetric INT4 clamps to [-7, 7] (s = max|w|/7), INT8 to [-127, 127];
 *   J  a zero range gives scale 0 and all codes 0 (also when the fp32 scale
 *      underflows to 0).
 *
 * Precision: every step that produces a stored integer or a stored scale runs in
 * IEEE binary32 with round-to-nearest-even (built with -fno-fast-math
 * -ffp-contract=off; nearbyintf under the default FE_TONEAREST mode).  GEMM
 * references run in binary64.
 *
 * Layouts: row-major everywhere.  X[M][K], W[K][N], Y[M][N]; groups run along K.
 *
 * Status codes returned here are the oracle's own: 0 ok, 1 non-finite input,
 * 2 a scale that does not fit fp16, 3 an argument out of range.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OR_OK 0
#define OR_NONFINITE 1
#define OR_RANGE 2
#define OR_ARGS 3

/* ------------------------------------------------------------------------- */
/* binary16 and bfloat16, decoded and encoded from the IEEE 754 definitions. */
/* ------------------------------------------------------------------------- */

/* Value of a binary16 bit pattern: 1 sign, 5 exponent (bias 15), 10 fraction. */
float qgo_f16_to_f32(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1F;
    int f = h & 0x3FF;
    float v;
    if (e == 0x1F)
        v = f ? NAN : INFINITY;
    else if (e == 0)
        v = ldexpf((float)f, -24);              /* subnormal: f * 2^-24 */
    else
        v = ldexpf((float)(f + 1024), e - 25);  /* (1 + f/2^10) * 2^(e-15) */
    return sign ? -v : v;
}

/* Largest binary16 pattern whose magnitude does not exceed a (a >= 0, finite):
 * rounding toward zero.  Magnitudes at or above 65536 clamp to 65504 (0x7BFF). */
static uint16_t f16_trunc_mag(float a)
{
    if (a >= 65536.0f) return 0x7BFF;
    if (a >= 0x1p-14f) {
        int e;
        float m = frexpf(a, &e);        /* a = m * 2^e, m in [0.5, 1) */
        /* a = (1 + frac) * 2^(e-1); unbiased exponent e-1, biased e-1+15 */
        int be = e - 1 + 15;
        if (be >= 31) return 0x7BFF;
        /* fraction bits: (2m - 1) * 2^10, truncated */
        uint32_t frac = (uint32_t)((2.0f * m - 1.0f) * 1024.0f);
        return (uint16_t)((be << 10) | frac);
    }
    /* subnormal range: multiples of 2^-24 */
    return (uint16_t)(uint32_t)(a * 16777216.0f);
}

/* binary32 -> binary16, rounding toward +infinity. */
uint16_t qgo_f32_to_f16_ru(float x)
{
    if (isnan(x)) return 0x7E00;
    if (isinf(x)) return x > 0 ? 0x7C00 : 0xFC00;
    if (x == 0.0f) return signbit(x) ? 0x8000 : 0x0000;
    if (x > 0.0f) {
        uint16_t h = f16_trunc_mag(x);
        if (qgo_f16_to_f32(h) < x) h = (uint16_t)(h + 1); /* next pattern up; 0x7BFF+1 = +inf */
        return h;
    }
    /* negative: toward +infinity is toward zero in magnitude */
    return (uint16_t)(0x8000 | f16_trunc_mag(-x));
}

/* binary32 -> bfloat16 (the upper 16 bits of binary32), round to nearest, ties to even. */
uint16_t qgo_f32_to_bf16_rn(float x)
{
    uint32_t u;
    memcpy(&u, &x, 4);
    if (isnan(x)) return (uint16_t)((u >> 16) | 0x0040);
    uint32_t hi = u >> 16;
    uint32_t lo = u & 0xFFFF;
    if (lo > 0x8000 || (lo == 0x8000 && (hi & 1))) hi += 1; /* carries into the exponent */
    return (uint16_t)hi;
}

float qgo_bf16_to_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

static int clampi(int v, int lo, int hi) { return v < lo ? lo : (v > hi ? hi : v); }

/* W~[k][n] = W[k][n] * s[k] (reading H), or W itself when s is NULL. */
static float smoothed(const float* W, const float* s, int64_t N, int64_t k, int64_t n)
{
    float w = W[k * N + n];
    return s ? w * s[k] : w;
}

/* ------------------------------------------------------------------------- */
/* O1: group-wise asymmetric INT4 (affine quantization, per-group granularity) */
/* ------------------------------------------------------------------------- */
int qgo_quantize_w4_asym(const float* W, const float* s_smooth, int64_t K, int64_t N, int group,
                         uint8_t* codes, uint16_t* scales_f16, uint8_t* zeros)
{
    int64_t G = K / group;
    int status = OR_OK;
#pragma omp parallel for schedule(static) reduction(max : status)
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t g = 0; g < G; ++g) {
            float mn = 0.0f, mx = 0.0f; /* reading A: the range always contains 0 */
            int bad = 0;
            for (int i = 0; i < group; ++i) {
                float v = smoothed(W, s_smooth, N, g * group + i, n);
                if (!isfinite(v)) bad = 1;
                if (v < mn) mn = v;
                if (v > mx) mx = v;
            }
            if (bad) { status = status > OR_NONFINITE ? status : OR_NONFINITE; continue; }
            float r = mx - mn;
            float s32 = r / 15.0f;                    /* reading B */
            uint16_t s16 = qgo_f32_to_f16_ru(s32);    /* reading C */
            if (s32 > 65504.0f) { status = OR_RANGE; continue; }
            float s = qgo_f16_to_f32(s16);
            int z = 0;
            if (r == 0.0f) { s16 = 0; s = 0.0f; }
            else z = clampi((int)nearbyintf(-mn / s), 0, 15);
            scales_f16[g * N + n] = s16;
            zeros[g * N + n] = (uint8_t)z;
            for (int i = 0; i < group; ++i) {
                int64_t k = g * group + i;
                int q = 0;
                if (s != 0.0f) {
                    float v = smoothed(W, s_smooth, N, k, n);
                    q = clampi((int)nearbyintf(v / s) + z, 0, 15); /* reading D */
                }
                codes[k * N + n] = (uint8_t)q;
            }
        }
    }
    return status;
}

/* ------------------------------------------------------------------------- */
/* O1s: group-wise symmetric INT4 (z = 0, s = max|w|/7), codes in [-7, 7]      */
/* ------------------------------------------------------------------------- */
int qgo_quantize_w4_sym(const float* W, const float* s_smooth, int64_t K, int64_t N, int group,
                        int8_t* codes, float* scales)
{
    int64_t G = K / group;
    int status = OR_OK;
#pragma omp parallel for schedule(static) reduction(max : status)
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t g = 0; g < G; ++g) {
            float amax = 0.0f;
            int bad = 0;
            for (int i = 0; i < group; ++i) {
                float v = smoothed(W, s_smooth, N, g * group + i, n);
                if (!isfinite(v)) bad = 1;
                float a = fabsf(v);
                if (a > amax) amax = a;
            }
            if (bad) { status = status > OR_NONFINITE ? status : OR_NONFINITE; continue; }
            float s = amax / 7.0f;
            scales[g * N + n] = s;
            for (int i = 0; i < group; ++i) {
                int64_t k = g * group + i;
                int q = 0;
                if (s != 0.0f) q = clampi((int)nearbyintf(smoothed(W, s_smooth, N, k, n) / s), -7, 7);
                codes[k * N + n] = (int8_t)q;
            }
        }
    }
    return status;
}

/* ------------------------------------------------------------------------- */
/* O2: 8 nibbles per uint32 along K, low nibble first (reading E)              */
/* ------------------------------------------------------------------------- */
void qgo_pack_nibbles(const uint8_t* codes, int64_t K, int64_t N, uint32_t* packed)
{
#pragma omp parallel for schedule(static)
    for (int64_t kb = 0; kb < K / 8; ++kb)
        for (int64_t n = 0; n < N; ++n) {
            uint32_t w = 0;
            for (int i = 0; i < 8; ++i)
                w |= (uint32_t)(codes[(8 * kb + i) * N + n] & 0xF) << (4 * i);
            packed[kb * N + n] = w;
        }
}

void qgo_unpack_nibbles(const uint32_t* packed, int64_t K, int64_t N, uint8_t* codes)
{
    for (int64_t k = 0; k < K; ++k)
        for (int64_t n = 0; n < N; ++n)
            codes[k * N + n] = (uint8_t)((packed[(k / 8) * N + n] >> (4 * (k % 8))) & 0xF);
}

/* Nibble of packed weight (k, n). */
static int nib(const uint32_t* packed, int64_t N, int64_t k, int64_t n)
{
    return (int)((packed[(k / 8) * N + n] >> (4 * (k % 8))) & 0xF);
}

/* ------------------------------------------------------------------------- */
/* O3: W4A16 GEMM reference.  W_deq[k][n] = (q - z) * s (exact in binary64).   */
/* y[r][n] = sum_k X[m_r][k] * W_deq[k][n] and bound[r][n] = sum_k |X||W_deq|.  */
/* rows == NULL means every row; otherwise only rows[0..nrows) are computed.   */
/* ------------------------------------------------------------------------- */
static double w4_asym_deq(const uint32_t* packed, const uint16_t* scales, const uint8_t* zeros,
                          int64_t N, int group, int64_t k, int64_t n)
{
    int64_t g = k / group;
    int q = nib(packed, N, k, n);
    return (double)(q - (int)zeros[g * N + n]) * (double)qgo_f16_to_f32(scales[g * N + n]);
}

void qgo_gemm_w4a16_ref(const float* X, int64_t M, int64_t K, int64_t N, const uint32_t* packed,
                        const uint16_t* scales, const uint8_t* zeros, int group,
                        const int64_t* rows, int64_t nrows, double* y, double* bound)
{
    if (!rows) nrows = M;
    memset(y, 0, sizeof(double) * nrows * N);
    memset(bound, 0, sizeof(double) * nrows * N);
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) {
            double w = w4_asym_deq(packed, scales, zeros, N, group, k, n);
            for (int64_t r = 0; r < nrows; ++r) {
                double x = (double)X[(rows ? rows[r] : r) * K + k];
                y[r * N + n] += x * w;
                bound[r * N + n] += fabs(x) * fabs(w);
            }
        }
}

/* ------------------------------------------------------------------------- */
/* O4: SmoothQuant smoothing factors (reading G: from a calibration batch).    */
/* s_j = max_m|Xcal[m][j]|^alpha / max_n|W[j][n]|^(1-alpha); inv_s_j = 1/s_j.  */
/* alpha == 0.5 uses fp32 sqrt and division (both correctly rounded).          */
/* A zero statistic on either side gives s_j = 1.                              */
/* ------------------------------------------------------------------------- */
int qgo_smooth_scales(const float* Xcal, int64_t Mc, const float* W, int64_t K, int64_t N,
                      float alpha, float* s, float* inv_s)
{
    int status = OR_OK;
#pragma omp parallel for schedule(static) reduction(max : status)
    for (int64_t j = 0; j < K; ++j) {
        float ax = 0.0f, aw = 0.0f;
        for (int64_t m = 0; m < Mc; ++m) {
            float v = Xcal[m * K + j];
            if (!isfinite(v)) status = OR_NONFINITE;
            if (fabsf(v) > ax) ax = fabsf(v);
        }
        for (int64_t n = 0; n < N; ++n) {
            float v = W[j * N + n];
            if (!isfinite(v)) status = OR_NONFINITE;
            if (fabsf(v) > aw) aw = fabsf(v);
        }
        float sj;
        if (ax == 0.0f || aw == 0.0f)
            sj = 1.0f;
        else if (alpha == 0.5f)
            sj = sqrtf(ax) / sqrtf(aw);
        else
            sj = (float)(pow((double)ax, (double)alpha) / pow((double)aw, 1.0 - (double)alpha));
        s[j] = sj;
        inv_s[j] = 1.0f / sj;
    }
    return status;
}

/* ------------------------------------------------------------------------- */
/* O5: per-token dynamic symmetric INT8 activations after smoothing.           */
/* X~ = X * inv_s; t_m = max_j|X~[m][j]| / 127; q = clamp(round(X~/t_m), +-127) */
/* ------------------------------------------------------------------------- */
int qgo_smooth_quant_act_i8(const float* X, int64_t M, int64_t K, const float* inv_s,
                            int8_t* Xq, float* t)
{
    int status = OR_OK;
#pragma omp parallel for schedule(static) reduction(max : status)
    for (int64_t m = 0; m < M; ++m) {
        float a = 0.0f;
        for (int64_t j = 0; j < K; ++j) {
            float v = inv_s ? X[m * K + j] * inv_s[j] : X[m * K + j];
            if (!isfinite(v)) status = OR_NONFINITE;
            if (fabsf(v) > a) a = fabsf(v);
        }
        float tm = a / 127.0f;
        t[m] = tm;
        for (int64_t j = 0; j < K; ++j) {
            float v = inv_s ? X[m * K + j] * inv_s[j] : X[m * K + j];
            int q = 0;
            if (tm != 0.0f && isfinite(v)) q = clampi((int)nearbyintf(v / tm), -127, 127);
            Xq[m * K + j] = (int8_t)q;
        }
    }
    return status;
}

/* ------------------------------------------------------------------------- */
/* O6: per-output-channel symmetric INT8 weights on W~ = diag(s) W.            */
/* sw_n = max_k|W~[k][n]| / 127; q = clamp(round(W~/sw_n), +-127)             */
/* ------------------------------------------------------------------------- */
int qgo_quantize_w8_channel(const float* W, const float* s_smooth, int64_t K, int64_t N,
                            int8_t* Wq, float* sw)
{
    int status = OR_OK;
#pragma omp parallel for schedule(static) reduction(max : status)
    for (int64_t n = 0; n < N; ++n) {
        float a = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            float v = smoothed(W, s_smooth, N, k, n);
            if (!isfinite(v)) status = OR_NONFINITE;
            if (fabsf(v) > a) a = fabsf(v);
        }
        float s = a / 127.0f;
        sw[n] = s;
        for (int64_t k = 0; k < K; ++k) {
            int q = 0;
            float v = smoothed(W, s_smooth, N, k, n);
            if (s != 0.0f && isfinite(v)) q = clampi((int)nearbyintf(v / s), -127, 127);
            Wq[k * N + n] = (int8_t)q;
        }
    }
    return status;
}

/* ------------------------------------------------------------------------- */
/* O7: W8A8 GEMM.  acc = sum_k qx*qw (exact integer);                          */
/* Y = bf16_rn(((float)acc * t_m) * sw_n); reference = fp64 dot of the        */
/* dequantized operands (qx*t_m)(qw*sw_n) and its absolute-value bound.         */
/* acc, y_bf16, yref, bound are [nrows][N]; any of acc / y_bf16 may be NULL.   */
/* ------------------------------------------------------------------------- */
void qgo_gemm_w8a8(const int8_t* Xq, const float* t, int64_t M, int64_t K, const int8_t* Wq,
                   const float* sw, int64_t N, const int64_t* rows, int64_t nrows,
                   int32_t* acc, uint16_t* y_bf16, double* yref, double* bound)
{
    if (!rows) nrows = M;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n)
        for (int64_t r = 0; r < nrows; ++r) {
            int64_t m = rows ? rows[r] : r;
            int64_t a = 0;
            double y = 0.0, b = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                int qx = Xq[m * K + k], qw = Wq[k * N + n];
                a += (int64_t)qx * qw;
                double xd = (double)qx * (double)t[m], wd = (double)qw * (double)sw[n];
                y += xd * wd;
                b += fabs(xd) * fabs(wd);
            }
            if (acc) acc[r * N + n] = (int32_t)a;
            if (y_bf16) y_bf16[r * N + n] = qgo_f32_to_bf16_rn(((float)a * t[m]) * sw[n]);
            yref[r * N + n] = y;
            bound[r * N + n] = b;
        }
}

/* ------------------------------------------------------------------------- */
/* O8: W4A8 GEMM with per-group partial sums.                                  */
/* P[m][g][n] = sum_{k in g} qx*qw4 (exact integer, qw4 in [-7,7] stored as    */
/* two's-complement nibbles); Y = t_m * sum_g P * s_gn.  The reference is the  */
/* fp64 dot of (qx*t_m)(qw4*s_gn) and its absolute-value bound.                */
/* part is [nrows][K/group][N] or NULL.                                        */
/* y_bf16 (nullable) is the output as the workload defines it ("int32 per-     */
/* group partial sums scaled by the group scale in fp32; bf16 out", "LLM       */
/* inference cost: W8A8/W4A8 ...", sec. 2.2): in binary32, each partial       */
/* converted and multiplied by its group scale, the products summed over g in  */
/* ascending order, the sum multiplied by t_m, then rounded once to bf16.      */
/* ------------------------------------------------------------------------- */
void qgo_gemm_w4a8(const int8_t* Xq, const float* t, int64_t M, int64_t K, const uint32_t* packed,
                   const float* sg, int64_t N, int group, const int64_t* rows, int64_t nrows,
                   int32_t* part, double* yref, double* bound, uint16_t* y_bf16)
{
    if (!rows) nrows = M;
    int64_t G = K / group;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n)
        for (int64_t r = 0; r < nrows; ++r) {
            int64_t m = rows ? rows[r] : r;
            double y = 0.0, b = 0.0;
            float acc = 0.0f;
            for (int64_t g = 0; g < G; ++g) {
                int64_t p = 0;
                for (int i = 0; i < group; ++i) {
                    int64_t k = g * group + i;
                    int v = nib(packed, N, k, n);
                    int qw = v >= 8 ? v - 16 : v; /* two's-complement nibble */
                    int qx = Xq[m * K + k];
                    p += (int64_t)qx * qw;
                    double xd = (double)qx * (double)t[m], wd = (double)qw * (double)sg[g * N + n];
                    y += xd * wd;
                    b += fabs(xd) * fabs(wd);
                }
                if (part) part[(r * G + g) * N + n] = (int32_t)p;
                {
                    volatile float prod = (float)p * sg[g * N + n]; /* one binary32 rounding */
                    acc = acc + prod;
                }
            }
            if (y_bf16) y_bf16[r * N + n] = qgo_f32_to_bf16_rn(acc * t[m]);
            yref[r * N + n] = y;
            bound[r * N + n] = b;
        }
}

/* Plain fp64 product of unquantized operands (the "no quantization" sanity figure):
 * y[r][n] = sum_k X[m_r][k] * W[k][n]. */
void qgo_gemm_f64(const float* X, int64_t M, int64_t K, const float* W, int64_t N,
                  const int64_t* rows, int64_t nrows, double* y)
{
    if (!rows) nrows = M;
    memset(y, 0, sizeof(double) * nrows * N);
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) {
            double w = (double)W[k * N + n];
            for (int64_t r = 0; r < nrows; ++r)
                y[r * N + n] += (double)X[(rows ? rows[r] : r) * K + k] * w;
        }
}

/* ------------------------------------------------------------------------- */
/* AWQ: activation-aware per-input-channel scales for the INT4 weights.        */
/* "Quantization & Flash Attention -- LLM inference optimization (2)":          */
/*   sec. 2.1  the statistic: the mean magnitude E[|X_c|] of each input channel */
/*             over a small calibration batch;                                  */
/*   sec. 2.2  the equivalent transform X W = (X / s)(s W), s per input channel;*/
/*   sec. 2.3  s_c = mean(|X_c|)^alpha, alpha on a grid in [0, 1], chosen to    */
/*             minimise the MSE between X W and the quantized layer's output.   */
/* Readings where the page is silent, each taken as stated here:              */
/*   L  the mean is a binary64 sum over the tokens in order, divided by the     */
/*      token count in binary64 and rounded once to binary32;                   */
/*   M  s_c = xm_c^alpha in binary64 (pow), rounded once to binary32; a channel */
/*      whose statistic is 0 keeps s_c = 1; inv_s_c = 1/s_c in binary32;       */
/*   N  the quantizer Q of sec. 2.3 acts on the scaled weight s W (the method   */
/*      quantizes weights only): asymmetric INT4 groups of O1 applied to        */
/*      diag(s) W, and the scaled activations X / s are stored in the layer's   */
/*      activation dtype: X~ = bf16_rn(X * inv_s);                              */
/*   O  the grid is alpha_i = i / (n_grid - 1), i = 0 .. n_grid - 1, both ends  */
/*      included (n_grid == 1: alpha = 0 only); the MSE is the mean over all    */
/*      M x N outputs of (X W - X~ deq(Q(s W)))^2 in binary64, both products    */
/*      exact up to binary64 rounding; the first grid point with the least MSE  */
/*      wins.                                                                   */
/* ------------------------------------------------------------------------- */

/* xm[c] = mean_m |X[m][c]| (reading L) */
void qgo_awq_act_mean(const float* X, int64_t M, int64_t K, float* xm)
{
#pragma omp parallel for schedule(static)
    for (int64_t c = 0; c < K; ++c) {
        double sum = 0.0;
        for (int64_t m = 0; m < M; ++m) sum += fabs((double)X[m * K + c]);
        xm[c] = (float)(sum / (double)M);
    }
}

/* s[c] = xm[c]^alpha, inv_s[c] = 1 / s[c] (reading M) */
void qgo_awq_scales(const float* xm, int64_t K, double alpha, float* s, float* inv_s)
{
    for (int64_t c = 0; c < K; ++c) {
        float sc = xm[c] == 0.0f ? 1.0f : (float)pow((double)xm[c], alpha);
        s[c] = sc;
        inv_s[c] = 1.0f / sc;
    }
}

/* X~[m][k] = bf16_rn(X[m][k] * inv_s[k]) as bf16 bit patterns (reading N) */
void qgo_awq_scale_act(const float* X, int64_t M, int64_t K, const float* inv_s, uint16_t* xs_bf16)
{
    for (int64_t m = 0; m < M; ++m)
        for (int64_t k = 0; k < K; ++k) xs_bf16[m * K + k] = qgo_f32_to_bf16_rn(X[m * K + k] * inv_s[k]);
}

/* grid point i of n (reading O) */
double qgo_awq_alpha(int i, int n_grid) { return n_grid > 1 ? (double)i / (double)(n_grid - 1) : 0.0; }

/* yref[m][n] = sum_k X[m][k] W[k][n] in binary64 */
static void awq_yref(const float* X, int64_t M, int64_t K, const float* W, int64_t N, double* yref)
{
    memset(yref, 0, sizeof(double) * M * N);
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) {
            double w = (double)W[k * N + n];
            for (int64_t m = 0; m < M; ++m) yref[m * N + n] += (double)X[m * K + k] * w;
        }
}

/* MSE of one candidate scale vector against yref (readings N, O).  Returns the
 * quantizer's status; *mse is left unset unless that status is 0. */
int qgo_awq_candidate_mse(const float* X, int64_t M, int64_t K, const float* W, int64_t N, int group,
                          const float* s, const float* inv_s, const double* yref, double* mse)
{
    uint8_t* codes = (uint8_t*)malloc((size_t)K * N);
    uint16_t* sc = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)(K / group) * N);
    uint8_t* z = (uint8_t*)malloc((size_t)(K / group) * N);
    float* xs = (float*)malloc(sizeof(float) * (size_t)M * K);
    double* yq = (double*)calloc((size_t)M * N, sizeof(double));
    int status = qgo_quantize_w4_asym(W, s, K, N, group, codes, sc, z); /* Q(diag(s) W), O1 */
    if (status == OR_OK) {
        for (int64_t m = 0; m < M; ++m)
            for (int64_t k = 0; k < K; ++k) /* X~ = bf16_rn(X * inv_s) */
                xs[m * K + k] = qgo_bf16_to_f32(qgo_f32_to_bf16_rn(X[m * K + k] * inv_s[k]));  /* = qgo_awq_scale_act */
#pragma omp parallel for schedule(static)
        for (int64_t n = 0; n < N; ++n)
            for (int64_t k = 0; k < K; ++k) {
                int64_t g = k / group;
                double w = (double)((int)codes[k * N + n] - (int)z[g * N + n]) * (double)qgo_f16_to_f32(sc[g * N + n]);
                for (int64_t m = 0; m < M; ++m) yq[m * N + n] += (double)xs[m * K + k] * w;
            }
        double acc = 0.0;
        for (int64_t i = 0; i < M * N; ++i) {
            double d = yref[i] - yq[i];
            acc += d * d;
        }
        *mse = acc / (double)(M * N);
    }
    free(codes);
    free(sc);
    free(z);
    free(xs);
    free(yq);
    return status;
}

/* The grid search of sec. 2.3: mse[i] for every grid point, *best = the first
 * index with the least MSE, and the scales at that point.  Returns the first
 * non-zero quantizer status (mse and best are then unspecified). */
int qgo_awq_search(const float* X, int64_t M, int64_t K, const float* W, int64_t N, int group, int n_grid,
                   double* mse, int* best, float* s_best, float* inv_s_best)
{
    float* xm = (float*)malloc(sizeof(float) * (size_t)K);
    float* s = (float*)malloc(sizeof(float) * (size_t)K);
    float* inv_s = (float*)malloc(sizeof(float) * (size_t)K);
    double* yref = (double*)malloc(sizeof(double) * (size_t)M * N);
    int status = OR_OK;
    qgo_awq_act_mean(X, M, K, xm);
    awq_yref(X, M, K, W, N, yref);
    int bi = 0;
    for (int i = 0; i < n_grid && status == OR_OK; ++i) {
        qgo_awq_scales(xm, K, qgo_awq_alpha(i, n_grid), s, inv_s);
        status = qgo_awq_candidate_mse(X, M, K, W, N, group, s, inv_s, yref, &mse[i]);
        if (status == OR_OK && mse[i] < mse[bi]) bi = i;
    }
    if (status == OR_OK) {
        *best = bi;
        qgo_awq_scales(xm, K, qgo_awq_alpha(bi, n_grid), s_best, inv_s_best);
    }
    free(xm);
    free(s);
    free(inv_s);
    free(yref);
    return status;
}

/* ------------------------------------------------------------------------- */
/* INT8 outlier side path beside the INT4 groups.                              */
/* "LLM inference cost: W8A8/W4A8 ...", sec. 2.2, second technique: during     */
/* calibration the largest-magnitude 2% of each group's weights are found,      */
/* kept in INT8 apart from the INT4 tile, and multiplied on a side path whose   */
/* result is added to the INT4 product.                                         */
/* Readings where the page is silent, each taken as stated here:              */
/*   P  per (group g, column n) the outliers are the count = ceil(2% of the     */
/*      group size) weights (3 of 128) of largest |w|, ranked by |w|            */
/*      descending, equal |w| by smaller k; slot r holds rank r;                */
/*   Q  they are stored as symmetric INT8 with one fp32 scale per (g, n):       */
/*      s8 = max|outlier| / 127, code = clamp(round(w / s8), -127, 127) (ties   */
/*      to even; s8 == 0 -> codes 0), with the k offset inside the group (u8);  */
/*   R  the INT4 part is the asymmetric INT4 group quantization (O1) of W with   */
/*      the outliers replaced by 0;                                             */
/*   S  Y = X deq4(dense) + X deq8(outliers); the reference runs in binary64.   */
/* Layouts: idx u8 [G][count][N], codes8 i8 [G][count][N], s8 fp32 [G][N].      */
/* ------------------------------------------------------------------------- */

/* count of outliers per group (reading P): ceil(0.02 * group) */
int qgo_outlier_count(int group) { return (2 * group + 99) / 100; }

/* Splits W~ (= diag(s) W, or W) into the outliers (idx, codes8, s8) and the dense
 * remainder W_dense (fp32 [K][N], outliers set to 0).  Returns 1 on a non-finite
 * element (that group's outputs are then unspecified). */
int qgo_outlier_split(const float* W, const float* s_smooth, int64_t K, int64_t N, int group, int count,
                      uint8_t* idx, int8_t* codes8, float* s8, float* W_dense)
{
    int64_t G = K / group;
    int status = OR_OK;
    if (count < 0 || count > 64 || count > group) return OR_ARGS;
#pragma omp parallel for schedule(static) reduction(max : status)
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t g = 0; g < G; ++g) {
            int pick[64];
            for (int i = 0; i < group; ++i) {
                float v = smoothed(W, s_smooth, N, g * group + i, n);
                if (!isfinite(v)) status = OR_NONFINITE;
                W_dense[(g * group + i) * N + n] = v;
            }
            /* reading P: repeated selection of the largest remaining |w|, first k on ties */
            for (int r = 0; r < count; ++r) {
                int best = -1;
                float bm = -1.0f;
                for (int i = 0; i < group; ++i) {
                    int taken = 0;
                    for (int j = 0; j < r; ++j) taken |= pick[j] == i;
                    if (taken) continue;
                    float a = fabsf(smoothed(W, s_smooth, N, g * group + i, n));
                    if (a > bm) { bm = a; best = i; }
                }
                pick[r] = best;
            }
            /* reading Q: symmetric INT8 over the outliers of this group */
            float amax = count > 0 ? fabsf(smoothed(W, s_smooth, N, g * group + pick[0], n)) : 0.0f;
            float sc = amax / 127.0f;
            s8[g * N + n] = sc;
            for (int r = 0; r < count; ++r) {
                float v = smoothed(W, s_smooth, N, g * group + pick[r], n);
                int q = sc != 0.0f ? clampi((int)nearbyintf(v / sc), -127, 127) : 0;
                idx[(g * count + r) * N + n] = (uint8_t)pick[r];
                codes8[(g * count + r) * N + n] = (int8_t)q;
                W_dense[(g * group + pick[r]) * N + n] = 0.0f; /* reading R */
            }
        }
    }
    return status;
}

/* y = X deq4 + X deq8 (reading S) in binary64, and bound = |X| |deq4| + |X| |deq8|,
 * for the selected rows. */
void qgo_gemm_w4a16_outlier_ref(const float* X, int64_t M, int64_t K, int64_t N, const uint32_t* packed,
                                const uint16_t* scales, const uint8_t* zeros, int group, int count,
                                const uint8_t* idx, const int8_t* codes8, const float* s8,
                                const int64_t* rows, int64_t nrows, double* y, double* bound)
{
    qgo_gemm_w4a16_ref(X, M, K, N, packed, scales, zeros, group, rows, nrows, y, bound);
    if (!rows) nrows = M;
    int64_t G = K / group;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n)
        for (int64_t g = 0; g < G; ++g)
            for (int r = 0; r < count; ++r) {
                int64_t k = g * group + idx[(g * count + r) * N + n];
                double w = (double)codes8[(g * count + r) * N + n] * (double)s8[g * N + n];
                for (int64_t i = 0; i < nrows; ++i) {
                    double x = (double)X[(rows ? rows[i] : i) * K + k];
                    y[i * N + n] += x * w;
                    bound[i * N + n] += fabs(x) * fabs(w);
                }
            }
}

/* ------------------------------------------------------------------------- */
/* GPTQ: INT4 weights with Hessian-weighted error compensation.                */
/* "Quantization & Flash Attention -- LLM inference optimization (2)",          */
/*   sec. 3.1  the Optimal Brain Surgeon idea: when one weight is rounded, move */
/*             the weights not yet rounded to compensate;                       */
/*   sec. 3.2  H = (2/n) X^T X + lambda I over n calibration samples; the       */
/*             dimensions are rounded one after another and the error of each  */
/*             is spread over the later ones through the inverse Hessian;       */
/*   sec. 3.3  blocks of 128 and a Cholesky factor make it fast and stable.     */
/* Readings where the page is silent, each taken as stated here:              */
/*   T  H is formed in binary64 with lambda = damp * mean(diag((2/n) X^T X)),   */
/*      damp = 0.01 (the page: a small ridge); an all-zero diagonal gives       */
/*      lambda = damp;                                                          */
/*   U  the dimensions the page's loop walks are the input channels, i.e. the   */
/*      rows k = 0 .. K-1 of W[K][N]; every output column n is rounded on its   */
/*      own, with the same compensation coefficients;                           */
/*   V  the grid is the stored INT4 format: asymmetric groups of `group` rows   */
/*      (O1's rules); a group's scale and zero come from its compensated        */
/*      weights, rounded to binary32, when the loop reaches the group's first   */
/*      row, and each row's code is O1's code of its compensated binary32 value;*/
/*   W  the update is the sequential OBS step in binary64: with Hinv the        */
/*      inverse Hessian over the rows not yet rounded,                          */
/*        e = (w_k - deq(q_k)) / Hinv[k][k];  w_j -= e * Hinv[k][j]  (j > k),   */
/*      then row and column k are eliminated from Hinv.  The Cholesky form of   */
/*      sec. 3.3 carries the same ratios Hinv[k][j] / Hinv[k][k] row by row.     */
/* ------------------------------------------------------------------------- */

/* Gauss-Jordan inverse in binary64.  H is symmetric positive definite (a Gram matrix
 * plus a positive ridge), so the elimination needs no pivoting: column c is scaled by
 * its pivot, then every other row r subtracts a[r][c] times row c (a[r][c] read before
 * the row changes).  Each product and difference is rounded on its own.  Returns 0, or 3
 * on a zero pivot. */
static int invert_f64(const double* A, int64_t n, double* inv)
{
    double* a = (double*)malloc(sizeof(double) * (size_t)n * n);
    double* f = (double*)malloc(sizeof(double) * (size_t)n);
    memcpy(a, A, sizeof(double) * (size_t)n * n);
    for (int64_t i = 0; i < n; ++i)
        for (int64_t j = 0; j < n; ++j) inv[i * n + j] = i == j ? 1.0 : 0.0;
    int status = OR_OK;
    for (int64_t c = 0; c < n && status == OR_OK; ++c) {
        double d = a[c * n + c];
        if (d == 0.0) { status = OR_ARGS; break; }
        for (int64_t j = 0; j < n; ++j) { a[c * n + j] /= d; inv[c * n + j] /= d; }
        for (int64_t r = 0; r < n; ++r) f[r] = a[r * n + c];
        for (int64_t r = 0; r < n; ++r) {
            if (r == c) continue;
            for (int64_t j = 0; j < n; ++j) {
                a[r * n + j] -= f[r] * a[c * n + j];
                inv[r * n + j] -= f[r] * inv[c * n + j];
            }
        }
    }
    free(a);
    free(f);
    return status;
}

/* H = (2/Mc) X^T X + lambda I (reading T), binary64, K x K. */
void qgo_gptq_hessian(const float* X, int64_t Mc, int64_t K, double damp, double* H)
{
#pragma omp parallel for schedule(static)
    for (int64_t a = 0; a < K; ++a)
        for (int64_t b = 0; b < K; ++b) {
            double s = 0.0;
            for (int64_t m = 0; m < Mc; ++m) s += (double)X[m * K + a] * (double)X[m * K + b];
            H[a * K + b] = 2.0 * s / (double)Mc;
        }
    double tr = 0.0;
    for (int64_t a = 0; a < K; ++a) tr += H[a * K + a];
    double lambda = tr > 0.0 ? damp * tr / (double)K : damp;
    for (int64_t a = 0; a < K; ++a) H[a * K + a] += lambda;
}

/* O1's scale and zero of one group of binary32 values (readings A-C, J).
 * Returns OR_RANGE when the scale does not fit fp16. */
static int asym_scale_zero(const float* v, int group, uint16_t* s16_out, float* s_out, int* z_out)
{
    float mn = 0.0f, mx = 0.0f;
    for (int i = 0; i < group; ++i) {
        if (v[i] < mn) mn = v[i];
        if (v[i] > mx) mx = v[i];
    }
    float r = mx - mn;
    float s32 = r / 15.0f;
    uint16_t s16 = qgo_f32_to_f16_ru(s32);
    float s = qgo_f16_to_f32(s16);
    int z = 0;
    if (r == 0.0f) { s16 = 0; s = 0.0f; }
    else z = clampi((int)nearbyintf(-mn / s), 0, 15);
    *s16_out = s16;
    *s_out = s;
    *z_out = z;
    return s32 > 65504.0f ? OR_RANGE : OR_OK;
}

/* GPTQ of W[K][N] against calibration X[Mc][K] -> O1-format codes, fp16 scales, zeros.
 * Returns 0, 1 on a non-finite weight, 2 on a scale above fp16, 3 on a singular H. */
int qgo_gptq(const float* X, int64_t Mc, int64_t K, const float* W, int64_t N, int group, double damp,
             uint8_t* codes, uint16_t* scales, uint8_t* zeros)
{
    int64_t G = K / group;
    double* H = (double*)malloc(sizeof(double) * (size_t)K * K);
    double* Hinv = (double*)malloc(sizeof(double) * (size_t)K * K);
    double* Wc = (double*)malloc(sizeof(double) * (size_t)K * N);
    float* gv = (float*)malloc(sizeof(float) * (size_t)group);
    float* sN = (float*)malloc(sizeof(float) * (size_t)N);
    int* zN = (int*)malloc(sizeof(int) * (size_t)N);
    int status = OR_OK;
    for (int64_t i = 0; i < K * N; ++i) {
        if (!isfinite(W[i])) status = OR_NONFINITE;
        Wc[i] = (double)W[i];
    }
    qgo_gptq_hessian(X, Mc, K, damp, H);
    if (status == OR_OK) status = invert_f64(H, K, Hinv);
    for (int64_t k = 0; k < K && status == OR_OK; ++k) {
        if (k % group == 0) { /* reading V: the group's scale and zero, from its compensated weights */
            int64_t g = k / group;
            for (int64_t n = 0; n < N; ++n) {
                for (int i = 0; i < group; ++i) gv[i] = (float)Wc[(k + i) * N + n];
                uint16_t s16;
                if (asym_scale_zero(gv, group, &s16, &sN[n], &zN[n]) != OR_OK) status = OR_RANGE;
                scales[g * N + n] = s16;
                zeros[g * N + n] = (uint8_t)zN[n];
            }
        }
        double d = Hinv[k * K + k];
        for (int64_t n = 0; n < N; ++n) {
            float w = (float)Wc[k * N + n];
            float s = sN[n];
            int z = zN[n];
            int q = s != 0.0f ? clampi((int)nearbyintf(w / s) + z, 0, 15) : 0;
            codes[k * N + n] = (uint8_t)q;
            double e = (Wc[k * N + n] - (double)(q - z) * (double)s) / d; /* reading W */
            for (int64_t j = k + 1; j < K; ++j) Wc[j * N + n] -= e * Hinv[k * K + j];
        }
        /* eliminate row and column k from the inverse Hessian of the remaining rows */
        for (int64_t a = k + 1; a < K; ++a) {
            double f = Hinv[a * K + k] / d;
            for (int64_t b = k + 1; b < K; ++b) Hinv[a * K + b] -= f * Hinv[k * K + b];
        }
    }
    free(H);
    free(Hinv);
    free(Wc);
    free(gv);
    free(sN);
    free(zN);
    return status;
}

/* Replays a given GPTQ result (codes, fp16 scales, zeros; e.g. one made on the GPU)
 * through the compensation of readings T-W, taking every decision from the arguments
 * (teacher forcing), so that one rounding difference does not change the rest of the
 * trajectory.  Reports:
 *   *code_slack   the largest distance, in grid steps, by which a given code lies
 *                 outside the rounding cell of its replayed value (0 when every code
 *                 is O1's code of its replayed binary32 value);
 *   *scale_miss   groups whose given scale differs from O1's scale of the replayed
 *                 group by more than `scale_ulps` fp16 units in the last place;
 *   *zero_miss    groups whose given zero differs from O1's zero by more than 1.
 * Returns the status of qgo_gptq's Hessian step (3 on a singular H). */
int qgo_gptq_replay(const float* X, int64_t Mc, int64_t K, const float* W, int64_t N, int group, double damp,
                    const uint8_t* codes, const uint16_t* scales, const uint8_t* zeros, int scale_ulps,
                    double* code_slack, int64_t* scale_miss, int64_t* zero_miss)
{
    double* H = (double*)malloc(sizeof(double) * (size_t)K * K);
    double* Hinv = (double*)malloc(sizeof(double) * (size_t)K * K);
    double* Wc = (double*)malloc(sizeof(double) * (size_t)K * N);
    float* gv = (float*)malloc(sizeof(float) * (size_t)group);
    for (int64_t i = 0; i < K * N; ++i) Wc[i] = (double)W[i];
    qgo_gptq_hessian(X, Mc, K, damp, H);
    int status = invert_f64(H, K, Hinv);
    double slack = 0.0;
    int64_t smiss = 0, zmiss = 0;
    for (int64_t k = 0; k < K && status == OR_OK; ++k) {
        int64_t g = k / group;
        if (k % group == 0)
            for (int64_t n = 0; n < N; ++n) {
                for (int i = 0; i < group; ++i) gv[i] = (float)Wc[(k + i) * N + n];
                uint16_t s16;
                float s_ref;
                int z_ref;
                asym_scale_zero(gv, group, &s16, &s_ref, &z_ref);
                if (abs((int)s16 - (int)scales[g * N + n]) > scale_ulps) ++smiss;
                if (abs(z_ref - (int)zeros[g * N + n]) > 1) ++zmiss;
            }
        double d = Hinv[k * K + k];
        for (int64_t n = 0; n < N; ++n) {
            float s = qgo_f16_to_f32(scales[g * N + n]);
            int z = zeros[g * N + n];
            int q = codes[k * N + n];
            float w = (float)Wc[k * N + n];
            int q_ref = s != 0.0f ? clampi((int)nearbyintf(w / s) + z, 0, 15) : 0;
            if (q != q_ref && s != 0.0f) {
                double t = (double)w / (double)s + (double)z; /* the replayed value in grid steps */
                double lo = q == 0 ? -INFINITY : (double)q - 0.5, hi = q == 15 ? INFINITY : (double)q + 0.5;
                double miss = t < lo ? lo - t : (t > hi ? t - hi : 0.0);
                if (miss > slack) slack = miss;
                if (miss == 0.0 && slack == 0.0) slack = 1e-300; /* a tie decided the other way */
            } else if (q != q_ref) {
                slack = INFINITY; /* a nonzero code in an all-zero group */
            }
            double e = (Wc[k * N + n] - (double)(q - z) * (double)s) / d;
            for (int64_t j = k + 1; j < K; ++j) Wc[j * N + n] -= e * Hinv[k * K + j];
        }
        for (int64_t a = k + 1; a < K; ++a) {
            double f = Hinv[a * K + k] / d;
            for (int64_t b = k + 1; b < K; ++b) Hinv[a * K + b] -= f * Hinv[k * K + b];
        }
    }
    *code_slack = slack;
    *scale_miss = smiss;
    *zero_miss = zmiss;
    free(H);
    free(Hinv);
    free(Wc);
    free(gv);
    return status;
}

/* ------------------------------------------------------------------------- */
/* 2:4 structured sparsity + INT4.                                              */
/* "LLM inference cost: W8A8/W4A8 ...", sec. 3.2: in every 4 weights the 2      */
/* largest are kept (2:4, the pattern the tensor cores accelerate), then the    */
/* kept weights are quantized to INT4 in groups of 128 with a zero point.       */
/* Readings where the page is silent, each taken as stated here:              */
/*   X  the 4-blocks run along K (the reduction dimension, as the hardware's    */
/*      2:4 pattern does), k = 4b .. 4b+3 of one column; "largest" is by |w|;   */
/*      ties go to the smaller k;                                               */
/*   Y  the INT4 step is O1 on the pruned matrix (groups of 128 along K; with   */
/*      reading A the pruned zeros do not change a group's range), and pruned   */
/*      positions dequantize to exactly 0 (they are not stored);                */
/*   Z  storage: the kept codes in k order, 8 per uint32 along K (vals          */
/*      [K/16][N], two per 4-block); the kept positions i0 < i1 of block b as   */
/*      the nibble (i1 << 2) | i0 at bits 4(b mod 8) of meta[b / 8][n]          */
/*      ([K/32][N]); fp16 scales and u8 zeros as O1.                            */
/* ------------------------------------------------------------------------- */

/* Wp = W with the 2 smaller |w| of every 4-block along K set to 0; meta as reading Z.
 * Requires K % 32 == 0. */
void qgo_prune24(const float* W, int64_t K, int64_t N, float* Wp, uint32_t* meta)
{
    memset(meta, 0, sizeof(uint32_t) * (size_t)(K / 32) * N);
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n)
        for (int64_t b = 0; b < K / 4; ++b) {
            /* the two largest |w| of the block, first k on ties */
            int keep[2] = {-1, -1};
            for (int r = 0; r < 2; ++r) {
                float best = -1.0f;
                for (int i = 0; i < 4; ++i) {
                    if (i == keep[0]) continue;
                    float a = fabsf(W[(4 * b + i) * N + n]);
                    if (a > best) { best = a; keep[r] = i; }
                }
            }
            int i0 = keep[0] < keep[1] ? keep[0] : keep[1];
            int i1 = keep[0] < keep[1] ? keep[1] : keep[0];
            for (int i = 0; i < 4; ++i) {
                float v = W[(4 * b + i) * N + n];
                Wp[(4 * b + i) * N + n] = (i == i0 || i == i1) ? v : 0.0f;
            }
            meta[(b / 8) * N + n] |= (uint32_t)((i1 << 2) | i0) << (4 * (b % 8));
        }
}

/* vals[kv/8][n] nibble kv%8 = the kv-th kept code of column n in k order (reading Z). */
void qgo_pack24_vals(const uint8_t* codes, const uint32_t* meta, int64_t K, int64_t N, uint32_t* vals)
{
    memset(vals, 0, sizeof(uint32_t) * (size_t)(K / 16) * N);
    for (int64_t n = 0; n < N; ++n)
        for (int64_t b = 0; b < K / 4; ++b) {
            uint32_t nib = (meta[(b / 8) * N + n] >> (4 * (b % 8))) & 0xF;
            int pos[2] = {(int)(nib & 3), (int)(nib >> 2)};
            for (int j = 0; j < 2; ++j) {
                int64_t kv = 2 * b + j;
                uint32_t c = codes[(4 * b + pos[j]) * N + n] & 0xF;
                vals[(kv / 8) * N + n] |= c << (4 * (kv % 8));
            }
        }
}

/* y = X * deq(sparse W) in binary64 and its |X||W| bound, for the selected rows. */
void qgo_gemm_w4a16_24_ref(const float* X, int64_t M, int64_t K, int64_t N, const uint32_t* vals,
                           const uint32_t* meta, const uint16_t* scales, const uint8_t* zeros, int group,
                           const int64_t* rows, int64_t nrows, double* y, double* bound)
{
    if (!rows) nrows = M;
    memset(y, 0, sizeof(double) * nrows * N);
    memset(bound, 0, sizeof(double) * nrows * N);
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n)
        for (int64_t b = 0; b < K / 4; ++b) {
            uint32_t nib = (meta[(b / 8) * N + n] >> (4 * (b % 8))) & 0xF;
            int pos[2] = {(int)(nib & 3), (int)(nib >> 2)};
            for (int j = 0; j < 2; ++j) {
                int64_t k = 4 * b + pos[j], kv = 2 * b + j, g = k / group;
                int q = (int)((vals[(kv / 8) * N + n] >> (4 * (kv % 8))) & 0xF);
                double w = (double)(q - (int)zeros[g * N + n]) * (double)qgo_f16_to_f32(scales[g * N + n]);
                for (int64_t r = 0; r < nrows; ++r) {
                    double x = (double)X[(rows ? rows[r] : r) * K + k];
                    y[r * N + n] += x * w;
                    bound[r * N + n] += fabs(x) * fabs(w);
                }
            }
        }
}
