/*
 * CPU oracle for the LLM.int8() mixed-precision linear layer -- declarations.
 * TEST INFRASTRUCTURE ONLY; see oracle.c.  fp16 values travel as their raw
 * binary16 bit patterns (uint16_t); every matrix is row-major and contiguous.
 */
#ifndef INT8ROW_ORACLE_H
#define INT8ROW_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

float    orc_half_to_float(uint16_t h);
uint16_t orc_double_to_half(double x);
float    orc_rhaz(float v);

void orc_quantize_weight_colwise(const uint16_t *W16, int K, int N,
                                 int8_t *Wq, float *sW);
int  orc_outlier_columns(const uint16_t *X, int T, int K, float alpha,
                         uint8_t *is_outlier, int32_t *idx);
void orc_outlier_hits(const uint16_t *X, int T, int K, float alpha, int32_t *hits);
float orc_frac_8bit(int count, int K);
void orc_quantize_rows(const uint16_t *X, int T, int K, const uint8_t *is_outlier,
                       int8_t *Xq, float *sX);
int  orc_int8_gemm(const int8_t *Xq, const int8_t *Wq, int T, int K, int N,
                   const int32_t *rows, int nrows, int32_t *acc);
void orc_dequantize_weight(const int8_t *Wq, const float *sW, int K, int N, uint16_t *W16d);
int  orc_mixed_linear(const uint16_t *X, int T, int K,
                      const int8_t *Wq, const float *sW, const uint16_t *W16, int N,
                      float alpha, const int32_t *rows, int nrows,
                      uint16_t *Y, double *Ypre, int32_t *acc_out);

void orc_int4_quantize_groupwise(const uint16_t *W16, int K, int N, int G,
                                 uint8_t *codes, uint16_t *scale, uint16_t *lo);
void orc_int4_dequantize(const uint8_t *codes, const uint16_t *scale, const uint16_t *lo,
                         int K, int N, int G, uint16_t *W16d);
void orc_int4_linear(const uint16_t *X, int T, int K, const uint8_t *codes,
                     const uint16_t *scale, const uint16_t *lo, int N, int G,
                     const int32_t *rows, int nrows, uint16_t *Y, double *Ypre);

#ifdef __cplusplus
}
#endif
#endif
