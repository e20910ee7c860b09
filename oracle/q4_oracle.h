/*
 * q4_oracle.h -- declarations of the plain C reference ("oracle") for the
 * weight-only 4-bit codebook linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  The test suite, the smoke check and the CPU
 * baseline leg of the benchmark are the only callers.  This header belongs to
 * the oracle alone: the CUDA library neither includes it nor links the oracle,
 * and the oracle includes nothing from the CUDA library.
 *
 * Conventions (shared meaning, separate code):
 *   W is logical [N][K] (out x in), y = x * W^T.
 *   codes  : uint8 [N][K/2], byte j of row n holds k = 2j in the low nibble
 *            and k = 2j+1 in the high nibble.
 *   scales : IEEE binary16 bit patterns [N][K/64], one per group of 64
 *            consecutive k of one row.
 *   cb     : 16 IEEE binary16 bit patterns (the codebook).
 *   x      : bfloat16 bit patterns [M][K];  y : float [M][N].
 */
#ifndef Q4_ORACLE_H
#define Q4_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ORACLE_GROUP 64

/* number formats */
float    oracle_h2f(uint16_t h);
uint16_t oracle_f2h_rne(float f);
float    oracle_bf2f(uint16_t b);
void     oracle_f2h_rne_array(const float* in, uint16_t* out, int64_t n);
void     oracle_h2f_array(const uint16_t* in, float* out, int64_t n);
void     oracle_bf2f_array(const uint16_t* in, float* out, int64_t n);

/* the NormalFloat-4 codebook, as 16 binary16 patterns in increasing order */
void     oracle_nf4_codebook(uint16_t cb[16]);
double   oracle_inv_phi(double p);

/* quantize W fp32 [N][K] to codes + scales; returns 0, or -1 on bad shape */
int      oracle_pack(const float* w, const uint16_t* cb, uint8_t* codes,
                     uint16_t* scales, int64_t N, int64_t K);

/* one weight of the quantized matrix, W[n][k] = cb[code] * scale in fp32 */
float    oracle_weight(const uint8_t* codes, const uint16_t* scales,
                       const uint16_t* cb, int64_t K, int64_t n, int64_t k);

/* explicit dense dequantization to fp32 [N][K]; returns 0 or -1 */
int      oracle_dequant(const uint8_t* codes, const uint16_t* scales,
                        const uint16_t* cb, float* w_out, int64_t N, int64_t K);

/* rows ids[i] of the dequantized matrix into out [n_ids][K]; ids outside
 * [0, N) give rows of zeros.  Returns 0 or -1. */
int      oracle_embed_rows(const uint8_t* codes, const uint16_t* scales,
                           const uint16_t* cb, const int32_t* ids, int64_t n_ids,
                           int64_t N, int64_t K, float* out);

/* y[m][i] = sum_k W[n_i][k] * x[m][k] in fp64, rounded once to fp32, and
 * absacc[m][i] = sum_k |W[n_i][k] * x[m][k]| in fp64.
 * rows == NULL: n_i = i for i < N and the outputs are [M][N];
 * otherwise n_i = rows[i] for i < nrows and the outputs are [M][nrows].
 * absacc may be NULL.  Returns 0 or -1. */
int      oracle_matmul(const uint8_t* codes, const uint16_t* scales,
                       const uint16_t* cb, const uint16_t* x, int64_t M,
                       int64_t N, int64_t K, const int64_t* rows, int64_t nrows,
                       float* y, double* absacc);

#ifdef __cplusplus
}
#endif
/* Two-bit variant (4-entry codebook cb4, codes [N][K/4], byte j holds
 * k = 4j + i in bits 2i, 2i+1; scales as the 4-bit format): pack, one weight,
 * dense dequantization, and the fp64 matmul (y [M][N], absacc may be NULL).
 * Each returns 0 or -1 for a bad shape, except oracle_weight2. */
int      oracle_pack2(const float* w, const uint16_t* cb4, uint8_t* codes,
                      uint16_t* scales, int64_t N, int64_t K);
float    oracle_weight2(const uint8_t* codes, const uint16_t* scales,
                        const uint16_t* cb4, int64_t K, int64_t n, int64_t k);
int      oracle_dequant2(const uint8_t* codes, const uint16_t* scales,
                         const uint16_t* cb4, float* w_out, int64_t N, int64_t K);
int      oracle_matmul2(const uint8_t* codes, const uint16_t* scales,
                        const uint16_t* cb4, const uint16_t* x, int64_t M,
                        int64_t N, int64_t K, float* y, double* absacc);

#endif
