/*
 * CPU oracle for the LLM.int8() mixed-precision linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may include, link,
 * load or call this file: only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg use it.  It shares no code, header, helper,
 * table or constant with the CUDA library; it has its own binary16
 * conversion, its own rounding and its own loops.
 *
 * Sources (web pages on the method):
 *   [P1] "LLM.int8()" abstract, taxoreview.com/v/2/lake/expert/dblp:280/8696
 *   [P2] "LLM.int8(): A Procedure for Int8 Matrix Multiplication in
 *        Transformer Language Models", summarizepaper.com/en/paper/2208.07339v1
 *        (sections "The LLM.int8() Methodology", summary bullets)
 *
 * What the pages fix: vector-wise quantisation, i.e. one normalisation
 * constant per row of X and one per output column of W, so that every inner
 * product has its own pair of constants [P1 abstract; P2 Methodology]; the
 * feature dimensions (columns of X) that carry outliers are split off and
 * multiplied in 16-bit together with the matching rows of W, everything
 * else is multiplied in 8-bit, and the two partial products are summed
 * [P1 abstract; P2 bullets 5-7].
 *
 * What the pages leave open, and the reading this oracle takes:
 *   - outlier rule: column k is an outlier when any |X[t,k]| >= alpha;
 *   - scale = absmax, code = clamp(rhaz(x * (127 / absmax)), -127, 127),
 *     with rhaz = round half away from zero, the reciprocal taken once in
 *     IEEE fp32 division and one fp32 multiply per element;
 *   - the row absmax is taken over the non-outlier columns only, and the
 *     outlier columns are zero in the int8 operand;
 *   - the column scale of W is taken over all K rows (conversion happens
 *     before any activation is seen);
 *   - the 16-bit part uses the fp16 W rows; accumulation is int32 for the
 *     8-bit part and (here) double for the 16-bit part and the merge;
 *   - the variant that keeps only Wq and sW resident (no fp16 weights; the
 *     memory-halving use of the method [P1 abstract]) takes the outlier rows
 *     of W dequantised: binary16 RNE of q * fl32(sW / 127), one fp32
 *     division per column and one fp32 multiply per element;
 *   - Y is rounded to binary16 with round-to-nearest-even.
 *
 * Quantisation decisions are taken in fp32, the precision the CUDA kernels
 * take them in, so the int8 codes must match bit for bit.  Everything that
 * is not a quantisation decision is done in double.
 *
 * The group-wise 4-bit weight codec (a second low-bit scheme on the pages:
 * the FlexGen summary, research.elamur.ai, "sheng-2023-flexgen", which states
 * that FlexGen compresses weights and the KV cache to 4 bits with group-wise
 * quantization and no retraining or calibration) is at the end of this file.
 * The page fixes neither the group, the code grid nor the rounding; the
 * readings taken are stated there.
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off -fno-fast-math -shared -fPIC.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include "oracle.h"

/* ------------------------------------------------------------------ */
/* IEEE-754 binary16 <-> binary32/64, written from the format definition. */
/* ------------------------------------------------------------------ */

/* binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
float orc_half_to_float(uint16_t h)
{
    uint32_t sign = (h >> 15) & 1u;
    uint32_t expo = (h >> 10) & 0x1fu;
    uint32_t frac = h & 0x3ffu;
    double mag;
    if (expo == 0) {
        mag = ldexp((double)frac, -24);                 /* subnormal: frac * 2^-24 */
    } else if (expo == 31) {
        mag = frac ? NAN : INFINITY;
    } else {
        mag = ldexp((double)(frac | 0x400u), (int)expo - 25); /* (1024+frac) * 2^(e-25) */
    }
    return (float)(sign ? -mag : mag);
}

/* Round-to-nearest, ties to even, of a non-negative double that holds an
 * exact multiple of a power of two (the caller has already scaled it). */
static double rne_nonneg(double q)
{
    double fl = floor(q);
    double diff = q - fl;                 /* exact: q and fl share an exponent range */
    if (diff > 0.5) return fl + 1.0;
    if (diff < 0.5) return fl;
    return (fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;
}

uint16_t orc_double_to_half(double x)
{
    uint16_t sign = signbit(x) ? 0x8000u : 0u;
    if (isnan(x)) return 0x7e00u;
    double a = fabs(x);
    /* largest finite binary16 is 65504; the midpoint to the next power of two
     * (65536, not representable) is 65520 and rounds to infinity (tie goes to
     * the even neighbour, which is 2^16). */
    if (a >= 65520.0) return sign | 0x7c00u;
    if (a < ldexp(1.0, -14)) {
        /* subnormal range: quantum 2^-24; n == 1024 carries into the smallest normal */
        double n = rne_nonneg(ldexp(a, 24));
        return sign | (uint16_t)n;
    }
    int e2;
    frexp(a, &e2);                        /* a = f * 2^e2, f in [0.5, 1) -> exponent e2-1 */
    int unbiased = e2 - 1;
    double n = rne_nonneg(ldexp(a, 10 - unbiased));   /* in [1024, 2048] */
    uint32_t bits = ((uint32_t)(unbiased + 15) << 10) + (uint32_t)(n - 1024.0);
    return sign | (uint16_t)bits;         /* n == 2048 carries into the exponent */
}

/* ------------------------------------------------------------------ */
/* Rounding rule shared by every quantiser.               */
/* ------------------------------------------------------------------ */

/* Round half away from zero, from the definition: take the integer part, and
 * step one unit away from zero when the discarded part is at least one half.
 * v - truncf(v) is exact in fp32 for every finite v. */
float orc_rhaz(float v)
{
    float r = truncf(v);
    if (fabsf(v - r) >= 0.5f) r += copysignf(1.0f, v);
    return r;
}

/* One element's int8 code given the reciprocal 127/absmax. */
static int8_t quantise_one(float x, float inv)
{
    float v = x * inv;                    /* one fp32 multiply, round to nearest */
    float r = orc_rhaz(v);
    if (r > 127.0f) r = 127.0f;
    if (r < -127.0f) r = -127.0f;
    return (int8_t)r;
}

static float reciprocal_127(float absmax)
{
    return absmax > 0.0f ? 127.0f / absmax : 0.0f;   /* IEEE fp32 division */
}

/* ------------------------------------------------------------------ */
/* a0. Weight conversion: one absmax per output column of W [P1, P2].   */
/* ------------------------------------------------------------------ */

void orc_quantize_weight_colwise(const uint16_t *W16, int K, int N,
                                 int8_t *Wq, float *sW)
{
    #pragma omp parallel for schedule(static)
    for (int n = 0; n < N; ++n) {
        float m = 0.0f;
        for (int k = 0; k < K; ++k) {
            float a = fabsf(orc_half_to_float(W16[(size_t)k * N + n]));
            if (a > m) m = a;
        }
        sW[n] = m;
        float inv = reciprocal_127(m);
        for (int k = 0; k < K; ++k)
            Wq[(size_t)k * N + n] = quantise_one(orc_half_to_float(W16[(size_t)k * N + n]), inv);
    }
}

/* ------------------------------------------------------------------ */
/* a1. Outlier feature dimensions: columns of X with any |x| >= alpha.  */
/* ------------------------------------------------------------------ */

int orc_outlier_columns(const uint16_t *X, int T, int K, float alpha,
                        uint8_t *is_outlier, int32_t *idx)
{
    for (int k = 0; k < K; ++k) is_outlier[k] = 0;
    for (int t = 0; t < T; ++t)
        for (int k = 0; k < K; ++k)
            if (fabsf(orc_half_to_float(X[(size_t)t * K + k])) >= alpha)
                is_outlier[k] = 1;
    int count = 0;
    for (int k = 0; k < K; ++k)
        if (is_outlier[k]) idx[count++] = k;      /* ascending */
    return count;
}

/* Per-column number of rows whose entry reaches alpha. */
void orc_outlier_hits(const uint16_t *X, int T, int K, float alpha, int32_t *hits)
{
    for (int k = 0; k < K; ++k) hits[k] = 0;
    for (int t = 0; t < T; ++t)
        for (int k = 0; k < K; ++k)
            if (fabsf(orc_half_to_float(X[(size_t)t * K + k])) >= alpha)
                hits[k] += 1;
}

/* Share of X's values that go through the 8-bit product: 1 - |O|/K. */
float orc_frac_8bit(int count, int K)
{
    return (float)(1.0 - (double)count / (double)K);
}

/* ------------------------------------------------------------------ */
/* a2. Row quantisation of the non-outlier part.      */
/* ------------------------------------------------------------------ */

static void quantise_row(const uint16_t *xrow, int K, const uint8_t *is_outlier,
                         int8_t *qrow, float *s_out)
{
    float m = 0.0f;
    for (int k = 0; k < K; ++k) {
        if (is_outlier[k]) continue;
        float a = fabsf(orc_half_to_float(xrow[k]));
        if (a > m) m = a;
    }
    *s_out = m;
    float inv = reciprocal_127(m);
    for (int k = 0; k < K; ++k)
        qrow[k] = is_outlier[k] ? 0 : quantise_one(orc_half_to_float(xrow[k]), inv);
}

void orc_quantize_rows(const uint16_t *X, int T, int K, const uint8_t *is_outlier,
                       int8_t *Xq, float *sX)
{
    #pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t)
        quantise_row(X + (size_t)t * K, K, is_outlier, Xq + (size_t)t * K, &sX[t]);
}

/* ------------------------------------------------------------------ */
/* a4. The 8-bit product, int32 accumulation checked against int64.     */
/* ------------------------------------------------------------------ */

/* acc[r, n] = sum_k Xq[rows[r], k] * Wq[k, n] for the listed rows.
 * Returns 0 when every int32 accumulator equals the int64 sum, -1 otherwise. */
int orc_int8_gemm(const int8_t *Xq, const int8_t *Wq, int T, int K, int N,
                  const int32_t *rows, int nrows, int32_t *acc)
{
    (void)T;
    int bad = 0;
    #pragma omp parallel for schedule(dynamic, 1) reduction(|:bad)
    for (int r = 0; r < nrows; ++r) {
        const int8_t *xq = Xq + (size_t)rows[r] * K;
        int64_t *s64 = (int64_t *)calloc((size_t)N, sizeof(int64_t));
        uint32_t *s32 = (uint32_t *)calloc((size_t)N, sizeof(uint32_t)); /* wraps mod 2^32 */
        for (int k = 0; k < K; ++k) {
            int32_t a = xq[k];
            if (a == 0) continue;
            const int8_t *wrow = Wq + (size_t)k * N;
            for (int n = 0; n < N; ++n) {
                int32_t p = a * (int32_t)wrow[n];
                s64[n] += p;
                s32[n] += (uint32_t)p;
            }
        }
        for (int n = 0; n < N; ++n) {
            int32_t v32 = (int32_t)s32[n];
            if (s64[n] > INT32_MAX || s64[n] < INT32_MIN || (int64_t)v32 != s64[n]) bad = 1;
            acc[(size_t)r * N + n] = v32;
        }
        free(s64);
        free(s32);
    }
    return bad ? -1 : 0;
}

/* ------------------------------------------------------------------ */
/* Dequantised weight rows (the Wq-only variant's 16-bit operand).      */
/* ------------------------------------------------------------------ */

/* W16d[k, n] = binary16 RNE of the fp32 product q * d[n], d[n] = fl32(sW[n] / 127),
 * for K rows of N columns: the inverse of the weight conversion, rounded to
 * the 16-bit type the outlier product runs in.  sW[n] = 0 gives zeros. */
void orc_dequantize_weight(const int8_t *Wq, const float *sW, int K, int N, uint16_t *W16d)
{
    for (int k = 0; k < K; ++k)
        for (int n = 0; n < N; ++n) {
            float d = sW[n] / 127.0f;                       /* IEEE fp32 division */
            float v = (float)Wq[(size_t)k * N + n] * d;     /* one fp32 multiply */
            W16d[(size_t)k * N + n] = orc_double_to_half((double)v);
        }
}

/* ------------------------------------------------------------------ */
/* a1-a6 together: the whole method for a list of rows of Y.            */
/* ------------------------------------------------------------------ */

/* X [T,K] fp16, Wq [K,N] int8, sW [N], W16 [K,N] fp16 (only its outlier rows
 * are read; NULL: the Wq-only variant, which dequantises those rows of Wq).  The outlier set is found over ALL T rows (it is a property of
 * the feature dimension, not of one row); rows of Y are then independent, so
 * only the listed rows are computed.  Outputs, per listed row r:
 *   Y[r, n]    binary16 bits of the result,
 *   Ypre[r, n] the same value in double before the final rounding (nullable),
 *   acc[r, n]  the int32 accumulators (nullable).
 * Returns |O|, or -1 if an int32 accumulator disagreed with its int64 sum. */
int orc_mixed_linear(const uint16_t *X, int T, int K,
                     const int8_t *Wq, const float *sW, const uint16_t *W16, int N,
                     float alpha, const int32_t *rows, int nrows,
                     uint16_t *Y, double *Ypre, int32_t *acc_out)
{
    uint8_t *is_outlier = (uint8_t *)malloc((size_t)K);
    int32_t *idx = (int32_t *)malloc((size_t)K * sizeof(int32_t));
    int count = orc_outlier_columns(X, T, K, alpha, is_outlier, idx);

    int8_t *Xq = (int8_t *)malloc((size_t)nrows * K);
    float *sX = (float *)malloc((size_t)nrows * sizeof(float));
    for (int r = 0; r < nrows; ++r)
        quantise_row(X + (size_t)rows[r] * K, K, is_outlier, Xq + (size_t)r * K, &sX[r]);

    int32_t *acc = acc_out ? acc_out : (int32_t *)malloc((size_t)nrows * N * sizeof(int32_t));
    int32_t *ident = (int32_t *)malloc((size_t)nrows * sizeof(int32_t));
    for (int r = 0; r < nrows; ++r) ident[r] = r;
    int ok = orc_int8_gemm(Xq, Wq, nrows, K, N, ident, nrows, acc);

    #pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < nrows; ++r) {
        const uint16_t *xrow = X + (size_t)rows[r] * K;
        /* a5: the 16-bit part over the outlier columns, in double */
        double *y16 = (double *)calloc((size_t)N, sizeof(double));
        uint16_t *wdq = W16 ? NULL : (uint16_t *)malloc((size_t)N * sizeof(uint16_t));
        for (int j = 0; j < count; ++j) {
            int k = idx[j];
            double xv = (double)orc_half_to_float(xrow[k]);
            const uint16_t *wrow;
            if (W16) {
                wrow = W16 + (size_t)k * N;
            } else {
                orc_dequantize_weight(Wq + (size_t)k * N, sW, 1, N, wdq);
                wrow = wdq;
            }
            for (int n = 0; n < N; ++n)
                y16[n] += xv * (double)orc_half_to_float(wrow[n]);
        }
        free(wdq);
        /* a6: dequantise by the outer product of the two scales, then merge */
        for (int n = 0; n < N; ++n) {
            double y = (double)acc[(size_t)r * N + n] * (double)sX[r] * (double)sW[n] / 16129.0
                       + y16[n];
            if (Ypre) Ypre[(size_t)r * N + n] = y;
            Y[(size_t)r * N + n] = orc_double_to_half(y);
        }
        free(y16);
    }

    if (!acc_out) free(acc);
    free(ident);
    free(sX);
    free(Xq);
    free(idx);
    free(is_outlier);
    return ok == 0 ? count : -1;
}

/* ------------------------------------------------------------------ */
/* Group-wise 4-bit weight codec (FlexGen summary: weights compressed  */
/* to 4 bits group-wise, with no retraining or calibration).           */
/* ------------------------------------------------------------------ */
/*
 * Readings (the page gives no formula):
 *   - a group is G consecutive rows k of one output column n of W [K,N]
 *     (groups run along the reduction axis, so each inner product meets
 *     K/G groups of its own column);
 *   - asymmetric min-max codes: lo = min and hi = max of the group, 16 levels
 *     lo + q*s, q in 0..15, with s = (hi - lo)/15 (nothing is calibrated);
 *   - s is kept as binary16: s = half_rn( fl32( fl32(hi - lo) / 15 ) ), and lo,
 *     a weight of the group, is binary16 already;
 *   - the code: inv = fl32(1 / s) (0 when s == 0), then
 *     q = clamp(rhaz( fl32( fl32(w - lo) * inv ) ), 0, 15), every step an IEEE
 *     fp32 operation, so the GPU can take the same decisions bit for bit;
 *   - the decoded weight is binary16, rounded once from the exact q*s + lo;
 *   - the product uses the decoded weights with the activation as it is
 *     (binary16), summed here in double and rounded once to binary16.
 * Layout here: codes [K,N] one per byte; scale and lo [K/G,N] binary16 bits.
 */

void orc_int4_quantize_groupwise(const uint16_t *W16, int K, int N, int G,
                                 uint8_t *codes, uint16_t *scale, uint16_t *lo_out)
{
    int groups = K / G;
    #pragma omp parallel for schedule(static)
    for (int n = 0; n < N; ++n) {
        for (int g = 0; g < groups; ++g) {
            float lo = INFINITY, hi = -INFINITY;
            for (int k = g * G; k < (g + 1) * G; ++k) {
                float w = orc_half_to_float(W16[(size_t)k * N + n]);
                if (w < lo) lo = w;
                if (w > hi) hi = w;
            }
            float range = hi - lo;                                /* fp32 subtraction */
            uint16_t s16 = orc_double_to_half((double)(range / 15.0f));   /* fp32 division, then binary16 */
            float s = orc_half_to_float(s16);
            float inv = s > 0.0f ? 1.0f / s : 0.0f;               /* fp32 division */
            scale[(size_t)g * N + n] = s16;
            lo_out[(size_t)g * N + n] = orc_double_to_half((double)lo);   /* exact: lo is a weight */
            for (int k = g * G; k < (g + 1) * G; ++k) {
                float d = orc_half_to_float(W16[(size_t)k * N + n]) - lo;  /* fp32 subtraction */
                float r = orc_rhaz(d * inv);                      /* one fp32 multiply */
                if (r < 0.0f) r = 0.0f;
                if (r > 15.0f) r = 15.0f;
                codes[(size_t)k * N + n] = (uint8_t)r;
            }
        }
    }
}

/* W16d[k,n] = binary16 of q*s + lo for the group of row k (q*s + lo is exact in
 * double: every term is a multiple of 2^-24 below 2^21). */
void orc_int4_dequantize(const uint8_t *codes, const uint16_t *scale, const uint16_t *lo,
                         int K, int N, int G, uint16_t *W16d)
{
    for (int k = 0; k < K; ++k)
        for (int n = 0; n < N; ++n) {
            size_t gi = (size_t)(k / G) * N + n;
            double v = (double)codes[(size_t)k * N + n] * (double)orc_half_to_float(scale[gi])
                       + (double)orc_half_to_float(lo[gi]);
            W16d[(size_t)k * N + n] = orc_double_to_half(v);
        }
}

/* Y[r,n] = binary16 of sum_k X[rows[r],k] * W~[k,n] (double sums) for the listed
 * rows, W~ the decoded 4-bit weight; Ypre (nullable) the sums before rounding. */
void orc_int4_linear(const uint16_t *X, int T, int K, const uint8_t *codes,
                     const uint16_t *scale, const uint16_t *lo, int N, int G,
                     const int32_t *rows, int nrows, uint16_t *Y, double *Ypre)
{
    (void)T;
    uint16_t *Wd = (uint16_t *)malloc((size_t)K * N * sizeof(uint16_t));
    orc_int4_dequantize(codes, scale, lo, K, N, G, Wd);
    #pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < nrows; ++r) {
        const uint16_t *xrow = X + (size_t)rows[r] * K;
        double *y = (double *)calloc((size_t)N, sizeof(double));
        for (int k = 0; k < K; ++k) {
            double xv = (double)orc_half_to_float(xrow[k]);
            if (xv == 0.0) continue;
            const uint16_t *wrow = Wd + (size_t)k * N;
            for (int n = 0; n < N; ++n) y[n] += xv * (double)orc_half_to_float(wrow[n]);
        }
        for (int n = 0; n < N; ++n) {
            if (Ypre) Ypre[(size_t)r * N + n] = y[n];
            Y[(size_t)r * N + n] = orc_double_to_half(y[n]);
        }
        free(y);
    }
    free(Wd);
}
