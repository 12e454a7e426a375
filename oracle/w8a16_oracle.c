/*
 * CPU oracle for the W8A16 linear layer -- TEST INFRASTRUCTURE ONLY.
 *
 * This file is the plain, slow, obviously-correct restatement of what the
 * GPU path computes.  Only the test-suite, the smoke check and the
 * benchmark's CPU-baseline leg may load it; the product library never links
 * or calls it, and it shares no code, header or table with the CUDA path.
 *
 * Sources (web pages on int8 weight-only quantization):
 *  - TPU-MLIR ChatGLM2 W8A16 article ("Exploring INT8 deployment of ChatGLM2
 *    on BM1684X"), section 2 "quantization scheme": only the Linear-layer
 *    weights are quantized, per channel, to int8; at compute time they are
 *    dequantized back to F16; activations stay F16.
 *  - same article, section 3 "TPU-MLIR implementation": the weight
 *    R = 4096x27392 F16 becomes int8 plus an F16 scale vector.
 *  - same article, section 4 "backend performance": the op loads, casts
 *    INT8 to F16, multiplies by the scale, multiplies with the activation
 *    and stores the result (steps 1-5).
 *  - LightSeq 2020 slides, slides "quantization: clipping + symmetric":
 *    symmetric quantization with bound = max|W| and 2^(n-1)-1 = 127 levels
 *    on each side of zero.
 * Where the pages leave a step open the following readings are used (each
 * is listed with its reason in the design notes):
 *  - one scale per OUTPUT channel n (column of W[K,N]);
 *  - scale_n = fp16_rne( fp32( amax_n / 127 ) ), the division in IEEE fp32;
 *  - q = clamp( rne( W / s ), -127, 127 ) with s the STORED fp16 scale
 *    widened to fp32, the division in IEEE fp32, ties to even;
 *  - an all-zero column has s = +0 and q = 0;
 *  - Y = X . (q o s) computed in the factored form s_n * sum_k x_k q_kn
 *    (exact in real arithmetic), here in fp64, plus an optional fp16 bias;
 *    the result is returned in fp64 and NOT rounded to fp16.
 * Inputs are assumed finite (NaN/Inf in W or X are outside the contract).
 *
 * Build: gcc -O2 -std=c11 -fno-fast-math -ffp-contract=off -fPIC -shared
 * (no SIMD intrinsics, no threads, no blocking).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ---------------------------------------------------------------------
 * IEEE-754 binary16 <-> binary32, written from the format definition
 * (1 sign bit, 5 exponent bits with bias 15, 10 fraction bits; subnormals
 * kept; round to nearest, ties to even).
 * ------------------------------------------------------------------- */

float oracle_f16_to_f32(uint16_t h)
{
    uint32_t sign = (uint32_t)(h >> 15) & 1u;
    uint32_t exp = (uint32_t)(h >> 10) & 0x1Fu;
    uint32_t frac = (uint32_t)h & 0x3FFu;
    float mag;
    if (exp == 0) {
        /* zero or subnormal: frac * 2^-24, exact in binary32 */
        mag = ldexpf((float)frac, -24);
    } else if (exp == 31) {
        mag = frac ? NAN : INFINITY;
    } else {
        /* (1024 + frac) * 2^(exp - 25), exact in binary32 */
        mag = ldexpf((float)(1024u + frac), (int)exp - 25);
    }
    return sign ? -mag : mag;
}

uint16_t oracle_f32_to_f16(float f)
{
    uint32_t x;
    memcpy(&x, &f, sizeof x);
    uint16_t sign = (uint16_t)((x >> 16) & 0x8000u);
    uint32_t exp32 = (x >> 23) & 0xFFu;
    uint32_t man32 = x & 0x7FFFFFu;

    if (exp32 == 0xFFu) {                      /* Inf or NaN */
        return (uint16_t)(sign | 0x7C00u | (man32 ? 0x200u : 0u));
    }
    if (exp32 == 0 && man32 == 0) {
        return sign;                          /* signed zero */
    }
    /* value = m * 2^e with m an integer (24-bit for normals) */
    int32_t e;
    uint32_t m;
    if (exp32 == 0) {                          /* binary32 subnormal */
        m = man32;
        e = -149;
    } else {
        m = man32 | 0x800000u;
        e = (int32_t)exp32 - 150;
    }
    /* Target: binary16 value = M * 2^E, where for normals 1024 <= M < 2048
     * and E = exponent - 25 >= -24; subnormals have E = -24, M < 1024.
     * Find the binary16 exponent of |f|: floor(log2(m * 2^e)). */
    int32_t msb = 31;
    while (((m >> msb) & 1u) == 0u) {
        msb--;
    }
    int32_t log2v = msb + e;                   /* floor(log2 |f|) */
    int32_t E = log2v - 10;                    /* ulp exponent for a normal */
    if (E < -24) {
        E = -24;                               /* subnormal range: ulp 2^-24 */
    }
    /* M = round_half_even(m * 2^(e - E)) */
    int32_t shift = E - e;                     /* bits to drop (may be <= 0) */
    uint64_t M;
    if (shift <= 0) {
        M = (uint64_t)m << (uint32_t)(-shift);
    } else if (shift >= 40) {
        M = 0;                                 /* far below half an ulp */
    } else {
        uint64_t mm = m;
        uint64_t q = mm >> (uint32_t)shift;
        uint64_t rem = mm & ((1ull << (uint32_t)shift) - 1ull);
        uint64_t half = 1ull << (uint32_t)(shift - 1);
        if (rem > half || (rem == half && (q & 1ull))) {
            q += 1;
        }
        M = q;
    }
    /* Rounding may carry into the next binade. */
    if (M >= 2048u) {
        M >>= 1;
        E += 1;
    }
    if (M >= 1024u) {
        int32_t biased = E + 25;               /* exponent field */
        if (biased >= 31) {
            return (uint16_t)(sign | 0x7C00u);  /* overflow -> Inf */
        }
        return (uint16_t)(sign | ((uint32_t)biased << 10) | ((uint32_t)M - 1024u));
    }
    /* subnormal (E == -24), or zero after rounding */
    return (uint16_t)(sign | (uint32_t)M);
}

/* ---------------------------------------------------------------------
 * Per-output-channel symmetric int8 quantization of W[K,N] (row-major).
 * Step order as the pages give it: bound = max|W| over the channel, the
 * scale puts the bound on level 127, then every weight is divided by the
 * scale, rounded and clipped to the symmetric range.
 * ------------------------------------------------------------------- */

static void quantize_column(const float *col_vals, int64_t K, int8_t *q_col,
                            int64_t N, uint16_t *scale_out)
{
    float amax = 0.0f;
    for (int64_t k = 0; k < K; ++k) {
        float a = fabsf(col_vals[k]);
        if (a > amax) {
            amax = a;
        }
    }
    float s32 = amax / 127.0f;                 /* IEEE fp32 division */
    uint16_t s16 = oracle_f32_to_f16(s32);
    float s = oracle_f16_to_f32(s16);
    for (int64_t k = 0; k < K; ++k) {
        int32_t qi;
        if (s == 0.0f) {
            qi = 0;
        } else {
            float r = col_vals[k] / s;         /* IEEE fp32 division */
            float rr = nearbyintf(r);          /* default mode: ties to even */
            if (rr > 127.0f) {
                rr = 127.0f;
            }
            if (rr < -127.0f) {
                rr = -127.0f;
            }
            qi = (int32_t)rr;
        }
        q_col[k * N] = (int8_t)qi;
    }
    *scale_out = s16;
}

/* W fp32 [K,N] -> q int8 [K,N], scales fp16 bits [N].  col_buf: K floats. */
void oracle_quantize_f32(const float *W, int64_t K, int64_t N, int8_t *q,
                         uint16_t *scales, float *col_buf)
{
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; ++k) {
            col_buf[k] = W[k * N + n];
        }
        quantize_column(col_buf, K, q + n, N, &scales[n]);
    }
}

/* W fp16 bits [K,N]: widened exactly to fp32, then as above. */
void oracle_quantize_f16(const uint16_t *W, int64_t K, int64_t N, int8_t *q,
                         uint16_t *scales, float *col_buf)
{
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; ++k) {
            col_buf[k] = oracle_f16_to_f32(W[k * N + n]);
        }
        quantize_column(col_buf, K, q + n, N, &scales[n]);
    }
}

/* ---------------------------------------------------------------------
 * Y[M,N] = X[M,K] . dequant(q)[K,N] (+ bias), in fp64.
 *   Y[m,n] = s_n * sum_k X[m,k] * q[k,n] + bias_n
 * acc: N doubles of caller-provided scratch.  bias may be NULL.
 * ------------------------------------------------------------------- */
void oracle_linear(const uint16_t *X, const int8_t *q, const uint16_t *scales,
                   const uint16_t *bias, int64_t M, int64_t K, int64_t N,
                   double *Y, double *acc)
{
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            acc[n] = 0.0;
        }
        for (int64_t k = 0; k < K; ++k) {
            double x = (double)oracle_f16_to_f32(X[m * K + k]);
            const int8_t *qrow = q + k * N;
            for (int64_t n = 0; n < N; ++n) {
                acc[n] += x * (double)qrow[n];
            }
        }
        for (int64_t n = 0; n < N; ++n) {
            double y = acc[n] * (double)oracle_f16_to_f32(scales[n]);
            if (bias) {
                y += (double)oracle_f16_to_f32(bias[n]);
            }
            Y[m * N + n] = y;
        }
    }
}

/* ---------------------------------------------------------------------
 * Clipped symmetric quantization -- the calibration choices the LightSeq
 * 2020 slides evaluate ("fixed range clip" and "percentage clip" against
 * plain max|W|, slide "quantization: clipping + symmetric").  The bound
 * that is put on level 127 is, per channel n:
 *   fixed range:  bound_n = min( max_k |W[k,n]|, c )        (c >= 0, fp32)
 *   percentage:   bound_n = the r-th smallest |W[k,n]|,
 *                 r = clamp( ceil(p K), 1, K ) in IEEE double  (0 < p <= 1)
 * and then, as in the symmetric quantizer, S = fp16_rne(fp32(bound)/127)
 * and q = clamp(rne(W / S), -127, 127): weights beyond the bound land on
 * +-127.  c = +inf and p = 1 are the plain symmetric quantizer.
 * ------------------------------------------------------------------- */

static float clampf_range(float v, float lo, float hi);

static int compare_floats(const void *a, const void *b)
{
    float x = *(const float *)a, y = *(const float *)b;
    return (x > y) - (x < y);
}

/* The codes of one column for a given bound (the symmetric quantizer's
 * second half). */
static void codes_for_bound(const float *col_vals, int64_t K, float bound, int8_t *q_col,
                            int64_t N, uint16_t *scale_out)
{
    uint16_t s16 = oracle_f32_to_f16(bound / 127.0f);
    float s = oracle_f16_to_f32(s16);
    for (int64_t k = 0; k < K; ++k) {
        int32_t qi = 0;
        if (s != 0.0f) {
            float rr = nearbyintf(col_vals[k] / s);
            rr = clampf_range(rr, -127.0f, 127.0f);
            qi = (int32_t)rr;
        }
        q_col[k * N] = (int8_t)qi;
    }
    *scale_out = s16;
}

/* mode 0: fixed range (param = c); mode 1: percentage (param = p).
 * col_buf: K floats; sort_buf: K floats. */
static void quantize_clip_column(const float *col_vals, int64_t K, int mode, double param,
                                 int8_t *q_col, int64_t N, uint16_t *scale_out, float *sort_buf)
{
    float bound = 0.0f;
    if (mode == 0) {
        for (int64_t k = 0; k < K; ++k) {
            float mag = fabsf(col_vals[k]);
            if (mag > bound) {
                bound = mag;
            }
        }
        float cf = (float)param;               /* the clip is an fp32 value */
        if (bound > cf) {
            bound = cf;
        }
    } else {
        double rr = ceil(param * (double)K);
        int64_t r = rr < 1.0 ? 1 : (rr > (double)K ? K : (int64_t)rr);
        for (int64_t k = 0; k < K; ++k) {
            sort_buf[k] = fabsf(col_vals[k]);
        }
        qsort(sort_buf, (size_t)K, sizeof(float), compare_floats);
        bound = sort_buf[r - 1];
    }
    codes_for_bound(col_vals, K, bound, q_col, N, scale_out);
}

/* W fp32 [K,N] or fp16 bits [K,N] (w_is_f16) -> q int8 [K,N], scales. */
void oracle_quantize_clip(const void *W, int w_is_f16, int64_t K, int64_t N, int mode, double param,
                          int8_t *q, uint16_t *scales, float *col_buf, float *sort_buf)
{
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; ++k) {
            col_buf[k] = w_is_f16 ? oracle_f16_to_f32(((const uint16_t *)W)[k * N + n])
                                  : ((const float *)W)[k * N + n];
        }
        quantize_clip_column(col_buf, K, mode, param, q + n, N, &scales[n], sort_buf);
    }
}

/* ---------------------------------------------------------------------
 * Outlier split -- the observation of the GOBO page applied to W8A16: the
 * few largest-magnitude weights of a channel inflate its scale, so they are
 * kept apart, exactly (as fp16), and the rest is quantized with the scale
 * of the remaining range.  Per channel n, with bound_n the r-th smallest
 * |W[k,n]|, r = clamp(ceil(p K), 1, K) in IEEE double (the percentage
 * clip's bound):
 *   outliers: every k with |W[k,n]| > bound_n, in increasing k; each kept
 *             as (k, fp16_rne(W[k,n])) and given the code 0;
 *   the rest: S = fp16_rne(fp32(bound_n)/127), q = clamp(rne(W/S), -127, 127).
 * At most cap = K - r weights of a channel are outliers (cap = 0 for p = 1,
 * the plain symmetric quantizer).  The side list is stored per channel in
 * cap slots: count[n], rows[n*cap + j], vals[n*cap + j] (unused slots 0).
 *   Y[m,n] = S_n sum_k X[m,k] q[k,n] + sum_j X[m, rows_j] vals_j + bias_n
 * ------------------------------------------------------------------- */

void oracle_quantize_outliers(const void *W, int w_is_f16, int64_t K, int64_t N, double p,
                              int8_t *q, uint16_t *scales, int32_t *count, int32_t *rows,
                              uint16_t *vals, float *col_buf, float *sort_buf)
{
    double rr = ceil(p * (double)K);
    int64_t r = rr < 1.0 ? 1 : (rr > (double)K ? K : (int64_t)rr);
    int64_t cap = K - r;
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; ++k) {
            col_buf[k] = w_is_f16 ? oracle_f16_to_f32(((const uint16_t *)W)[k * N + n])
                                  : ((const float *)W)[k * N + n];
            sort_buf[k] = fabsf(col_buf[k]);
        }
        qsort(sort_buf, (size_t)K, sizeof(float), compare_floats);
        float cut = sort_buf[r - 1];
        codes_for_bound(col_buf, K, cut, q + n, N, &scales[n]);
        int32_t c = 0;
        for (int64_t j = 0; j < cap; ++j) {
            rows[n * cap + j] = 0;
            vals[n * cap + j] = 0;
        }
        for (int64_t k = 0; k < K; ++k) {
            /* at most K - r magnitudes exceed the r-th smallest, so c < cap
             * always holds; the test only keeps every write inside the slots */
            if (fabsf(col_buf[k]) > cut && c < cap) {
                rows[n * cap + c] = (int32_t)k;
                vals[n * cap + c] = oracle_f32_to_f16(col_buf[k]);
                q[k * N + n] = 0;
                ++c;
            }
        }
        count[n] = c;
    }
}

/* Y[M,N] = X . dequant(q) + X . outliers (+ bias), in fp64. */
void oracle_linear_outliers(const uint16_t *X, const int8_t *q, const uint16_t *scales,
                            const int32_t *count, const int32_t *rows, const uint16_t *vals,
                            int64_t cap, const uint16_t *bias, int64_t M, int64_t K, int64_t N,
                            double *Y, double *acc)
{
    oracle_linear(X, q, scales, bias, M, K, N, Y, acc);
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            double extra = 0.0;
            for (int32_t j = 0; j < count[n]; ++j) {
                extra += (double)oracle_f16_to_f32(X[m * K + rows[n * cap + j]]) *
                         (double)oracle_f16_to_f32(vals[n * cap + j]);
            }
            Y[m * N + n] += extra;
        }
    }
}

/* ---------------------------------------------------------------------
 * Asymmetric (affine) per-output-channel int8 quantization -- the variant
 * the LightSeq 2020 slides set against the symmetric one (slide
 * "quantization: clipping + symmetric": a weight is (i - z) S, and the
 * product of two such values expands into four integer terms), with the
 * range, scale and zero point of the integer-arithmetic quantization paper
 * those slides cite (arXiv 1712.05877, section 2):
 *   lo = min(0, min_k W), hi = max(0, max_k W)   (0 stays representable)
 *   S  = fp16_rne( fp32(hi - lo) / 255 )          (256 levels, -128..127)
 *   z  = clamp( rne( -128 - lo / S ), -128, 127 )
 *   q  = clamp( rne( W / S ) + z, -128, 127 )
 * every operation in IEEE fp32 with S the stored fp16 value widened; an
 * all-zero column has S = 0, z = 0 and q = 0.  Dequantized: (q - z) S.
 * ------------------------------------------------------------------- */

static float clampf_range(float v, float lo, float hi)
{
    if (v < lo) {
        return lo;
    }
    if (v > hi) {
        return hi;
    }
    return v;
}

static void quantize_column_asym(const float *col_vals, int64_t K, int8_t *q_col,
                                 int64_t N, uint16_t *scale_out, int8_t *zero_out)
{
    float lo = 0.0f, hi = 0.0f;
    for (int64_t k = 0; k < K; ++k) {
        if (col_vals[k] < lo) {
            lo = col_vals[k];
        }
        if (col_vals[k] > hi) {
            hi = col_vals[k];
        }
    }
    float range = hi - lo;                       /* IEEE fp32 subtraction */
    uint16_t s16 = oracle_f32_to_f16(range / 255.0f);
    float s = oracle_f16_to_f32(s16);
    int32_t z = 0;
    if (s != 0.0f) {
        float t = lo / s;
        float zf = nearbyintf(-128.0f - t);      /* ties to even */
        z = (int32_t)clampf_range(zf, -128.0f, 127.0f);
    }
    for (int64_t k = 0; k < K; ++k) {
        int32_t qi = 0;
        if (s != 0.0f) {
            float rr = nearbyintf(col_vals[k] / s);
            /* |W / S| stays far below 2^20 (S >= the smallest fp16
             * subnormal whenever it is non-zero); the bound only keeps the
             * conversion defined */
            rr = clampf_range(rr, -1048576.0f, 1048576.0f);
            qi = (int32_t)rr + z;
            if (qi > 127) {
                qi = 127;
            }
            if (qi < -128) {
                qi = -128;
            }
        }
        q_col[k * N] = (int8_t)qi;
    }
    *scale_out = s16;
    *zero_out = (int8_t)z;
}

/* W fp32 [K,N] -> q int8 [K,N], scales fp16 bits [N], zeros int8 [N]. */
void oracle_quantize_asym_f32(const float *W, int64_t K, int64_t N, int8_t *q,
                              uint16_t *scales, int8_t *zeros, float *col_buf)
{
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; ++k) {
            col_buf[k] = W[k * N + n];
        }
        quantize_column_asym(col_buf, K, q + n, N, &scales[n], &zeros[n]);
    }
}

void oracle_quantize_asym_f16(const uint16_t *W, int64_t K, int64_t N, int8_t *q,
                              uint16_t *scales, int8_t *zeros, float *col_buf)
{
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; ++k) {
            col_buf[k] = oracle_f16_to_f32(W[k * N + n]);
        }
        quantize_column_asym(col_buf, K, q + n, N, &scales[n], &zeros[n]);
    }
}

/* Y[m,n] = S_n * sum_k X[m,k] * (q[k,n] - z_n) + bias_n, in fp64. */
void oracle_linear_asym(const uint16_t *X, const int8_t *q, const uint16_t *scales,
                        const int8_t *zeros, const uint16_t *bias, int64_t M,
                        int64_t K, int64_t N, double *Y, double *acc)
{
    for (int64_t row = 0; row < M; ++row) {
        for (int64_t col = 0; col < N; ++col) {
            acc[col] = 0.0;
        }
        for (int64_t k = 0; k < K; ++k) {
            double xv = (double)oracle_f16_to_f32(X[row * K + k]);
            const int8_t *codes = q + k * N;
            for (int64_t col = 0; col < N; ++col) {
                acc[col] += xv * (double)((int32_t)codes[col] - (int32_t)zeros[col]);
            }
        }
        for (int64_t col = 0; col < N; ++col) {
            double out = acc[col] * (double)oracle_f16_to_f32(scales[col]);
            if (bias) {
                out += (double)oracle_f16_to_f32(bias[col]);
            }
            Y[row * N + col] = out;
        }
    }
}

/* Element-wise array forms of the two conversions (used by the pins). */
void oracle_f32_to_f16_array(const float *src, int64_t n, uint16_t *dst)
{
    for (int64_t i = 0; i < n; ++i) {
        dst[i] = oracle_f32_to_f16(src[i]);
    }
}

void oracle_f16_to_f32_array(const uint16_t *src, int64_t n, float *dst)
{
    for (int64_t i = 0; i < n; ++i) {
        dst[i] = oracle_f16_to_f32(src[i]);
    }
}
