/*
 * lbq_oracle.h -- plain, slow, fp64 CPU reference of the low-bit weight formats
 * and products. TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the
 * bench's CPU-baseline leg call it; the product path never does. It shares no
 * code, header, table or constant generator with the CUDA library.
 *
 * Formats (ids 1 = ternary 5-trits-per-byte, 2 = 1-bit sign, 3 = 2-bit with
 * rotated input) are described where they are implemented, in lbq_oracle.c.
 * Every function returns 0 on success and a negative number on bad arguments.
 */
#ifndef LBQ_ORACLE_H
#define LBQ_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* IEEE 754 binary16 from binary64, round to nearest even; overflow -> inf. */
uint16_t orc_f16_from_f64(double v);
double orc_f16_to_f64(uint16_t h);
double orc_bf16_to_f64(uint16_t b);

/* Packed sizes: bytes per code row, fp16 scales per row, weights per scale. */
int orc_layout(int fmt, int64_t K, int64_t* code_stride, int64_t* scale_stride,
               int64_t* block);

/* Quantise + pack W [N][K] fp32. scales may be NULL for fmt 1 (scales in-block). */
int orc_pack(int fmt, const float* W, int64_t K, int64_t N, uint8_t* codes,
             uint16_t* scales);

/* Unpack to integer codes (t, 2b-1 or q) [N][K] and block scales [N][K/block]
 * (as fp64). Returns -2 if a byte is not a valid code (e.g. a ternary byte
 * above 242 or non-zero padding trits). */
int orc_unpack(int fmt, const uint8_t* codes, const uint16_t* scales, int64_t K,
               int64_t N, int8_t* out, double* block_scales);

/* Dequantised weights [N][K] in fp64. */
int orc_dequant(int fmt, const uint8_t* codes, const uint16_t* scales, int64_t K,
                int64_t N, double* What);

/* SplitMix64 sign vector: D[k] = -1 iff the top bit of output k+1 is set. */
int orc_rht_signs(uint64_t seed, int64_t K, int8_t* D);
/* Raw SplitMix64 outputs (for pinning the generator). */
int orc_splitmix64(uint64_t seed, int64_t n, uint64_t* out);

/* x' = H_512 D x / sqrt(512) per 512-block, fp64 in and out, [M][K]. */
int orc_hadamard(const double* x, const int8_t* D, int64_t M, int64_t K, double* out);

/* Y[m][n] = sum_k What[n][k] * xin[m][k] and Bnd[m][n] = sum_k |What[n][k] xin[m][k]|,
 * xin = X (bf16 bits -> fp64) or, for fmt 3, its rotation with D. Rows are split
 * over nthreads POSIX threads (the arithmetic per element is the same sequential
 * loop whatever nthreads is). Bnd may be NULL. */
int orc_gemm(int fmt, const uint8_t* codes, const uint16_t* scales, int64_t K, int64_t N,
             const uint16_t* X, int64_t M, const int8_t* D, double* Y, double* Bnd,
             int nthreads);

#ifdef __cplusplus
}
#endif

#endif
