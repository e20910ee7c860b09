/*
 * q4_oracle.c -- plain, slow, single-threaded reference ("oracle") for the
 * weight-only 4-bit codebook linear layer: pack (quantize), dequantize and
 * the matmul y = x * W^T with W rebuilt from codes, scales and codebook.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * CPU-baseline leg of the benchmark load this library.  It shares no code,
 * header, table or helper with the CUDA library, and includes nothing of it.
 *
 * Build: cc -std=c99 -O2 -ffp-contract=off -fPIC -shared q4_oracle.c -lm
 * (x86-64 SSE arithmetic, so every float operation below is one IEEE-754
 * binary32 operation rounded to nearest-even; no FMA contraction).
 *
 * What it follows:
 *  - "deep-fold" (github wertick01/deep-fold), section "Method": each group
 *    of 64 weights stores 4-bit NF4 codes and one FP16 scale; the packed
 *    payload is about 3.76x smaller than BF16; kernels rebuild the values as
 *    they multiply.  Same page, "Method" table: decode is a GEMV, prefill a
 *    tensor-core GEMM.
 *  - Same page, introduction and Figure 1: embeddings (PackedEmbed) decode
 *    only the requested rows, on a path of their own.
 *  - "Trapetum" overview, "What it does": the fused kernel decodes each
 *    weight from the codebook as it multiplies.  "Trapetum" landing page: the matrix is
 *    decoded inside the matmul and never materialized.
 *  - "Trapetum" overview, "In one sentence" and "Frontier models on your own
 *    hardware": a 70B model in 2 bits (the two-bit variant below).
 *  - NF4 (NormalFloat, QLoRA): sixteen quantiles of the standard normal,
 *    asymmetric (8 positive, 7 negative, an exact zero), scaled to [-1, 1].
 *
 * Readings taken where the pages are silent, stated once here:
 *  - groups run along K (64 consecutive k of one output row n);
 *  - scale = binary16(absmax of the group), rounded to nearest-even;
 *  - code = index of the codebook entry nearest to w / scale, the division and
 *    the distances |w/scale - cb_i| taken in binary32, scanned from i = 0 with a
 *    strict "<", so that a tie goes to the lowest index;
 *  - a scale that rounds to zero gives every weight of the group the index of
 *    the entry of smallest magnitude (the exact 0 of NF4);
 *  - nibble order: k = 2j in the low nibble of byte j, k = 2j+1 in the high;
 *  - dequantized weight W = cb[code] * scale in binary32 (exact: an 11-bit by
 *    11-bit significand product);
 *  - matmul reference: the products W * x summed in fp64 in increasing k and
 *    rounded once to binary32;
 *  - embedding rows: the requested rows of the dequantized matrix in binary32;
 *    an id outside [0, N) gives a row of zeros;
 *  - the two-bit variant (the pages name 2-bit codebooks, print none): the same
 *    steps with a 4-entry codebook and four codes per byte (see below).
 */
#include "q4_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* Number formats, written from the IEEE-754 binary16 / bfloat16 definitions */
/* ------------------------------------------------------------------------ */

/* binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits.
 * exponent 0 -> subnormal fraction * 2^-24; exponent 31 -> inf / NaN. */
float oracle_h2f(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1F;
    int frac = h & 0x3FF;
    double v;
    if (e == 0)
        v = ldexp((double)frac, -24);
    else if (e == 31)
        v = frac ? NAN : INFINITY;
    else
        v = ldexp((double)(frac + 1024), e - 25);
    return (float)(sign ? -v : v);
}

/* Round a double to the nearest binary16, ties to even, with subnormals and
 * overflow to infinity.  Used for binary32 inputs (exact in double) and for
 * the codebook construction. */
static uint16_t d2h_rne(double v)
{
    uint16_t sign = signbit(v) ? 0x8000u : 0u;
    double a = fabs(v);
    int e2, E;
    double q;
    if (isnan(v))
        return 0x7E00u;
    if (isinf(v))
        return (uint16_t)(sign | 0x7C00u);
    if (a == 0.0)
        return sign;
    frexp(a, &e2);          /* a = m * 2^e2, m in [0.5, 1) */
    E = e2 - 1;             /* a in [2^E, 2^(E+1)) */
    if (E < -14) {
        /* subnormal range: count units of 2^-24; q == 1024 is the encoding
         * of the smallest normal number, which is the right answer there */
        q = rint(ldexp(a, 24));
        return (uint16_t)(sign | (uint16_t)q);
    }
    q = rint(ldexp(a, 10 - E));   /* significand scaled to [1024, 2048] */
    if (q == 2048.0) {
        q = 1024.0;
        E += 1;
    }
    if (E > 15)
        return (uint16_t)(sign | 0x7C00u);
    return (uint16_t)(sign | (uint16_t)(((E + 15) << 10) | ((int)q - 1024)));
}

uint16_t oracle_f2h_rne(float f)
{
    return d2h_rne((double)f);
}

/* bfloat16 is the upper half of a binary32 pattern */
float oracle_bf2f(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

void oracle_f2h_rne_array(const float* in, uint16_t* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = oracle_f2h_rne(in[i]);
}

void oracle_h2f_array(const uint16_t* in, float* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = oracle_h2f(in[i]);
}

void oracle_bf2f_array(const uint16_t* in, float* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = oracle_bf2f(in[i]);
}

/* ------------------------------------------------------------------------ */
/* NF4 codebook                                                              */
/* ------------------------------------------------------------------------ */

/* Standard normal CDF Phi(q) = erfc(-q / sqrt 2) / 2, inverted by bisection. */
double oracle_inv_phi(double p)
{
    double lo = -40.0, hi = 40.0;
    for (int it = 0; it < 200; ++it) {
        double mid = 0.5 * (lo + hi);
        double cdf = 0.5 * erfc(-mid / sqrt(2.0));
        if (cdf < p)
            lo = mid;
        else
            hi = mid;
    }
    return 0.5 * (lo + hi);
}

/* NormalFloat-4 (QLoRA): quantiles of N(0,1) over two ranges, 9 equally
 * spaced probabilities from p_max down to 1/2 for the positive side and 8 for
 * the negative side; the probability 1/2 of each side is the shared zero,
 * kept once.  p_max = 1 - (1/(2*15) + 1/(2*16)) / 2, the mean of the two
 * sides' outer bin centres, keeps the extreme quantile finite.  All values
 * are divided by the largest magnitude, so the ends are exactly -1 and +1,
 * then rounded to binary16.  Output is in increasing order. */
void oracle_nf4_codebook(uint16_t cb[16])
{
    const double p_max = 1.0 - 0.5 * (1.0 / 30.0 + 1.0 / 32.0);
    double v[16];
    int n = 0;
    /* negative side, most negative first: 7 values */
    for (int i = 0; i < 7; ++i) {
        double p = p_max + (0.5 - p_max) * (double)i / 7.0;
        v[n++] = -oracle_inv_phi(p);
    }
    v[n++] = 0.0;
    /* positive side, smallest first: 8 values */
    for (int i = 7; i >= 0; --i) {
        double p = p_max + (0.5 - p_max) * (double)i / 8.0;
        v[n++] = oracle_inv_phi(p);
    }
    double vmax = oracle_inv_phi(p_max);
    for (int i = 0; i < 16; ++i)
        cb[i] = d2h_rne(v[i] / vmax);
}

/* ------------------------------------------------------------------------ */
/* Pack (quantize)                                                           */
/* ------------------------------------------------------------------------ */

static int nearest_code(float r, const float cbf[16])
{
    int best = 0;
    float bestd = fabsf(r - cbf[0]);
    for (int i = 1; i < 16; ++i) {
        float d = fabsf(r - cbf[i]);
        if (d < bestd) {
            bestd = d;
            best = i;
        }
    }
    return best;
}

int oracle_pack(const float* w, const uint16_t* cb, uint8_t* codes,
                uint16_t* scales, int64_t N, int64_t K)
{
    if (N < 0 || K <= 0 || K % ORACLE_GROUP != 0)
        return -1;
    float cbf[16];
    for (int i = 0; i < 16; ++i)
        cbf[i] = oracle_h2f(cb[i]);

    /* index of the entry of smallest magnitude, for zero scales */
    int zero_code = 0;
    for (int i = 1; i < 16; ++i)
        if (fabsf(cbf[i]) < fabsf(cbf[zero_code]))
            zero_code = i;

    const int64_t G = K / ORACLE_GROUP;
    int c[ORACLE_GROUP];
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t g = 0; g < G; ++g) {
            const float* wg = w + n * K + g * ORACLE_GROUP;
            float a = 0.0f;
            for (int j = 0; j < ORACLE_GROUP; ++j) {
                float m = fabsf(wg[j]);
                if (m > a)
                    a = m;
            }
            uint16_t sh = oracle_f2h_rne(a);
            float s = oracle_h2f(sh);
            scales[n * G + g] = sh;
            for (int j = 0; j < ORACLE_GROUP; ++j) {
                if (s == 0.0f) {
                    c[j] = zero_code;
                } else {
                    float r = wg[j] / s;
                    c[j] = nearest_code(r, cbf);
                }
            }
            uint8_t* cg = codes + n * (K / 2) + g * (ORACLE_GROUP / 2);
            for (int j = 0; j < ORACLE_GROUP / 2; ++j)
                cg[j] = (uint8_t)(c[2 * j] | (c[2 * j + 1] << 4));
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Dequantize                                                                */
/* ------------------------------------------------------------------------ */

float oracle_weight(const uint8_t* codes, const uint16_t* scales,
                    const uint16_t* cb, int64_t K, int64_t n, int64_t k)
{
    uint8_t byte = codes[n * (K / 2) + k / 2];
    int code = (k % 2 == 0) ? (byte & 0x0F) : (byte >> 4);
    float v = oracle_h2f(cb[code]);
    float s = oracle_h2f(scales[n * (K / ORACLE_GROUP) + k / ORACLE_GROUP]);
    return v * s;
}

int oracle_dequant(const uint8_t* codes, const uint16_t* scales,
                   const uint16_t* cb, float* w_out, int64_t N, int64_t K)
{
    if (N < 0 || K <= 0 || K % ORACLE_GROUP != 0)
        return -1;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k)
            w_out[n * K + k] = oracle_weight(codes, scales, cb, K, n, k);
    return 0;
}

/* Embedding rows ("deep-fold", introduction and Figure 1: embeddings decode
 * only the requested rows): out[i] = row ids[i] of the dequantized matrix,
 * a row of zeros for an id outside [0, N). */
int oracle_embed_rows(const uint8_t* codes, const uint16_t* scales,
                      const uint16_t* cb, const int32_t* ids, int64_t n_ids,
                      int64_t N, int64_t K, float* out)
{
    if (n_ids < 0 || N < 0 || K <= 0 || K % ORACLE_GROUP != 0)
        return -1;
    for (int64_t i = 0; i < n_ids; ++i) {
        int64_t n = ids[i];
        for (int64_t k = 0; k < K; ++k)
            out[i * K + k] = (n >= 0 && n < N) ? oracle_weight(codes, scales, cb, K, n, k) : 0.0f;
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Matmul: dequantize one row of W, then the fp64 dot product with each x    */
/* ------------------------------------------------------------------------ */

int oracle_matmul(const uint8_t* codes, const uint16_t* scales,
                  const uint16_t* cb, const uint16_t* x, int64_t M,
                  int64_t N, int64_t K, const int64_t* rows, int64_t nrows,
                  float* y, double* absacc)
{
    if (M < 0 || N < 0 || K <= 0 || K % ORACLE_GROUP != 0)
        return -1;
    int64_t nout = rows ? nrows : N;
    if (nout < 0)
        return -1;
    float* wrow = (float*)malloc((size_t)K * sizeof(float));
    if (!wrow)
        return -1;
    for (int64_t i = 0; i < nout; ++i) {
        int64_t n = rows ? rows[i] : i;
        if (n < 0 || n >= N) {
            free(wrow);
            return -1;
        }
        for (int64_t k = 0; k < K; ++k)
            wrow[k] = oracle_weight(codes, scales, cb, K, n, k);
        for (int64_t m = 0; m < M; ++m) {
            double acc = 0.0, aacc = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                double p = (double)wrow[k] * (double)oracle_bf2f(x[m * K + k]);
                acc += p;
                aacc += fabs(p);
            }
            y[m * nout + i] = (float)acc;
            if (absacc)
                absacc[m * nout + i] = aacc;
        }
    }
    free(wrow);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Two-bit variant: a 4-entry codebook, four codes per byte                  */
/* ------------------------------------------------------------------------ */
/* "Trapetum" overview, sections "In one sentence" and "Frontier models on
 * your own hardware": a 70B model in 2 bits; the pages print no 2-bit layout.
 * Reading: the 4-bit
 * format with 2-bit codes -- groups of 64 along K and one binary16 scale per
 * group (binary16 of the group's absmax, rounded to nearest-even); a code is
 * the index of the entry nearest to w / scale (binary32, ties to the lowest
 * index); a zero scale gives every weight the entry of smallest magnitude;
 * byte j of a row holds k = 4j + i in bits 2i and 2i + 1. */

static int nearest_of_four(float q, const float e[4])
{
    int pick = 0;
    float dist = fabsf(q - e[0]);
    for (int i = 1; i < 4; ++i) {
        float di = fabsf(q - e[i]);
        if (di < dist) {
            dist = di;
            pick = i;
        }
    }
    return pick;
}

int oracle_pack2(const float* w, const uint16_t* cb4, uint8_t* codes,
                 uint16_t* scales, int64_t N, int64_t K)
{
    if (N < 0 || K <= 0 || K % ORACLE_GROUP != 0)
        return -1;
    float e[4];
    for (int i = 0; i < 4; ++i)
        e[i] = oracle_h2f(cb4[i]);
    int least = 0;
    for (int i = 1; i < 4; ++i)
        if (fabsf(e[i]) < fabsf(e[least]))
            least = i;
    const int64_t G = K / ORACLE_GROUP;
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t g = 0; g < G; ++g) {
            const float* src = w + n * K + g * ORACLE_GROUP;
            float amax = 0.0f;
            for (int j = 0; j < ORACLE_GROUP; ++j) {
                float t = fabsf(src[j]);
                if (t > amax)
                    amax = t;
            }
            uint16_t sbits = oracle_f2h_rne(amax);
            float sv = oracle_h2f(sbits);
            scales[n * G + g] = sbits;
            uint8_t* dst = codes + n * (K / 4) + g * (ORACLE_GROUP / 4);
            for (int j = 0; j < ORACLE_GROUP / 4; ++j)
                dst[j] = 0;
            for (int j = 0; j < ORACLE_GROUP; ++j) {
                int code = (sv == 0.0f) ? least : nearest_of_four(src[j] / sv, e);
                dst[j / 4] = (uint8_t)(dst[j / 4] | (code << (2 * (j % 4))));
            }
        }
    }
    return 0;
}

float oracle_weight2(const uint8_t* codes, const uint16_t* scales,
                     const uint16_t* cb4, int64_t K, int64_t n, int64_t k)
{
    uint8_t b = codes[n * (K / 4) + k / 4];
    int code = (b >> (2 * (k % 4))) & 3;
    float val = oracle_h2f(cb4[code]);
    float sc = oracle_h2f(scales[n * (K / ORACLE_GROUP) + (k / ORACLE_GROUP)]);
    return val * sc;
}

int oracle_dequant2(const uint8_t* codes, const uint16_t* scales,
                    const uint16_t* cb4, float* w_out, int64_t N, int64_t K)
{
    if (N < 0 || K <= 0 || K % ORACLE_GROUP != 0)
        return -1;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t kk = 0; kk < K; ++kk)
            w_out[n * K + kk] = oracle_weight2(codes, scales, cb4, K, n, kk);
    return 0;
}

int oracle_matmul2(const uint8_t* codes, const uint16_t* scales,
                   const uint16_t* cb4, const uint16_t* x, int64_t M,
                   int64_t N, int64_t K, float* y, double* absacc)
{
    if (M < 0 || N < 0 || K <= 0 || K % ORACLE_GROUP != 0)
        return -1;
    float* row = (float*)malloc((size_t)K * sizeof(float));
    if (!row)
        return -1;
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t kk = 0; kk < K; ++kk)
            row[kk] = oracle_weight2(codes, scales, cb4, K, n, kk);
        for (int64_t m = 0; m < M; ++m) {
            double sum = 0.0, abs_sum = 0.0;
            for (int64_t kk = 0; kk < K; ++kk) {
                double prod = (double)row[kk] * (double)oracle_bf2f(x[m * K + kk]);
                sum += prod;
                abs_sum += fabs(prod);
            }
            y[m * N + n] = (float)sum;
            if (absacc)
                absacc[m * N + n] = abs_sum;
        }
    }
    free(row);
    return 0;
}
