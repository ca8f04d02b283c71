/*
 * oracle.h - plain CPU reference for the MoE low-precision quantization path.
 * TEST INFRASTRUCTURE: only tests, the smoke check and the benchmark's CPU
 * baseline use it. Independent of the CUDA library (no shared code).
 * All pointers are host pointers; bf16 inputs are passed as raw uint16 words.
 * Every function returns 0 on success or one of the ORACLE_ERR_* codes.
 */
#ifndef MXQ_ORACLE_H
#define MXQ_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ORACLE_FLOOR 0
#define ORACLE_RCEIL 1

#define ORACLE_ERR_ARG 1
#define ORACLE_ERR_OFFSETS 2

double oracle_e4m3_value(uint8_t code);
uint8_t oracle_e4m3_from_float(float v);
void oracle_e4m3_from_float_array(const float *v, int64_t n, uint8_t *out);
float oracle_fp8_scale(float amax);
float oracle_fp8_inv_scale(float amax);
uint8_t oracle_e8m0_floor(float amax);
uint8_t oracle_e8m0_rceil(float amax);
uint8_t oracle_e8m0(float amax, int mode);
uint8_t oracle_mx_element(float x, uint8_t scale_byte);
int64_t oracle_blocked_offset(int64_t r, int64_t c, int64_t cols_padded);
int64_t oracle_blocked_grouped_rows_bound(int64_t rows, int32_t groups);

int oracle_fp8_quant_jagged_rowwise(const uint16_t *in, int64_t rows, int64_t cols,
                                    int64_t stride_row, int64_t stride_col,
                                    const int32_t *offs, int32_t groups,
                                    uint8_t *out, float *inv_scales);
int oracle_fp8_quant_jagged_colwise(const uint16_t *in, int64_t rows, int64_t cols,
                                    int64_t stride_row, int64_t stride_col,
                                    const int32_t *offs, int32_t groups,
                                    uint8_t *out, float *inv_scales);
int oracle_fp8_quant_blockwise(const uint16_t *in, int64_t rows, int64_t cols,
                               int32_t br, int32_t bc, uint8_t *out, float *inv_scales);
int oracle_fp8_quant_blockwise_transposed(const uint16_t *in, int64_t rows, int64_t cols,
                                          int32_t br, int32_t bc, uint8_t *out, float *inv_scales);
int oracle_fp8_grouped_gemm_rowwise(const uint8_t *a, const float *inv_a, const uint8_t *w, const float *inv_w,
                                    int64_t M, int64_t N, int64_t K, const int32_t *offs, int32_t groups,
                                    double *out);
int oracle_mx_grouped_gemm(const uint8_t *a, const uint8_t *sa, const uint8_t *w, const uint8_t *sw,
                           int64_t M, int64_t N, int64_t K, const int32_t *offs, int32_t groups, double *out);
int64_t oracle_mx_jagged_blocks(const int32_t *offs, int32_t groups);
int oracle_mx_quant_jagged_colwise(const uint16_t *in, int64_t rows, int64_t cols, int64_t stride_row,
                                   int64_t stride_col, const int32_t *offs, int32_t groups, int mode, uint8_t *out,
                                   uint8_t *scales);
int oracle_mx_grouped_gemm_wgrad(const uint8_t *a, const uint8_t *sa, const uint8_t *b, const uint8_t *sb,
                                 int64_t N, int64_t K, int64_t M, const int32_t *offs, int32_t groups, double *out);
int oracle_fp8_grouped_gemm_wgrad(const uint8_t *a, const float *inv_a, const uint8_t *b, const float *inv_b,
                                  int64_t N, int64_t K, int64_t M, const int32_t *offs, int32_t groups,
                                  double *out);
int oracle_mx_quant_3d_colwise(const uint16_t *in, int64_t E, int64_t N, int64_t K,
                               int mode, uint8_t *out, uint8_t *scales);
int oracle_mx_quant_rowwise(const uint16_t *in, int64_t rows, int64_t cols, int mode,
                            uint8_t *out, uint8_t *scales);
int oracle_mx_scales_to_blocked_grouped(const uint8_t *scales, int64_t rows, int64_t cols,
                                        const int32_t *offs, int32_t groups,
                                        uint8_t *out, int64_t capacity_rows,
                                        int32_t *group_row_starts);
int64_t oracle_blocked_grouped_k_cols_bound(int64_t cols, int32_t groups);
int oracle_mx_scales_to_blocked_grouped_k(const uint8_t *scales, int64_t rows, int64_t cols,
                                          const int32_t *offs, int32_t groups,
                                          uint8_t *out, int64_t capacity_cols,
                                          int32_t *group_col_starts);
int oracle_mx_quant_rowwise_blocked_grouped(const uint16_t *in, int64_t rows, int64_t cols, int mode,
                                            const int32_t *offs, int32_t groups,
                                            uint8_t *out, uint8_t *scales_blocked,
                                            int64_t capacity_rows, int32_t *group_row_starts);

#ifdef __cplusplus
}
#endif

#endif
