/*
 * CPU oracle for the SmoothQuant W8A8 + per-request LoRA linear layer.
 * TEST INFRASTRUCTURE ONLY (tests, smoke check, CPU-baseline benchmark leg).
 * Independent of the CUDA library: no shared code, header or constants.
 *
 * Conventions: X is [M,K] row-major, f32 (dtype 0) or bf16 bit patterns
 * (dtype 1); W is [N,K] bf16 bits (output channels by input channels);
 * LoRA A is [r,K] and B is [N,r], bf16 bits.  All buffers are host memory
 * owned by the caller.
 */
#ifndef SQ_ORACLE_H
#define SQ_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { SQO_F32 = 0, SQO_BF16 = 1 };

int sqo_num_threads(void);
uint16_t sqo_round_bf16(float f);

void sqo_act_absmax_update(const void *X, int dtype, int64_t M, int64_t K, float *act_absmax);
void sqo_weight_absmax(const uint16_t *W, int64_t N, int64_t K, float *w_absmax);
void sqo_compute_smoothing(const float *act_absmax, const float *w_absmax, int64_t K,
                           float alpha, float *s);
void sqo_quantize_weight(const uint16_t *W, const float *s, int64_t N, int64_t K,
                         int8_t *Wq, float *w_scale);
void sqo_quant_act(const void *X, int dtype, const float *s, int64_t M, int64_t K,
                   int8_t *Xq, float *x_scale);
float sqo_static_act_scale(const float *act_absmax, const float *s, int64_t K);
int64_t sqo_quant_act_static(const void *X, int dtype, const float *s, float scale, int64_t M,
                             int64_t K, int8_t *Xq, float *x_scale);
void sqo_fold_norm_weight(const float *gamma, const float *s, int64_t K, float *gamma_s);
double sqo_sum_squares_bf16(const uint16_t *h, int64_t K);
void sqo_rmsnorm_quant_act(const uint16_t *H, const float *gamma_s, float eps, int64_t M,
                           int64_t K, int8_t *Xq, float *x_scale);
void sqo_prepare_lora(const uint16_t *A, const uint16_t *B, const float *s, int64_t r,
                      int64_t K, int64_t N, float lora_alpha, uint16_t *A_s,
                      uint16_t *B_s);
void sqo_gemm_rows(const int8_t *Xq, const int8_t *Wq, int64_t M, int64_t N, int64_t K,
                   const int64_t *rows, int64_t nrows, int64_t *acc);
void sqo_gemm_pairs(const int8_t *Xq, const int8_t *Wq, int64_t K, const int64_t *rows,
                    const int64_t *cols, int64_t npairs, int64_t *acc);
int sqo_token_adapter(const int32_t *seg_offsets, const int32_t *seg_adapter, int64_t S,
                      int n_adapters, int64_t i);
void sqo_linear_lora_rows(const int8_t *Xq, const float *x_scale, const int8_t *Wq,
                          const float *w_scale, int64_t M, int64_t N, int64_t K,
                          int n_adapters, const uint16_t *const *A_s,
                          const uint16_t *const *B_s, const int64_t *ranks,
                          const int32_t *seg_offsets, const int32_t *seg_adapter, int64_t S,
                          const int64_t *rows, int64_t nrows, double *Y, double *delta,
                          int64_t *acc);
void sqo_linear_lora_raw_rows(const uint16_t *X, const int8_t *Xq, const float *x_scale,
                              const int8_t *Wq, const float *w_scale, int64_t M, int64_t N,
                              int64_t K, int n_adapters, const uint16_t *const *A,
                              const uint16_t *const *B_s, const int64_t *ranks,
                              const int32_t *seg_offsets, const int32_t *seg_adapter,
                              int64_t S, const int64_t *rows, int64_t nrows, double *Y,
                              double *delta);
void sqo_reference_rows(const void *X, int dtype, const uint16_t *W, int64_t M, int64_t N,
                        int64_t K, int n_adapters, const uint16_t *const *A,
                        const uint16_t *const *B, const int64_t *ranks,
                        const double *lora_alpha, const int32_t *seg_offsets,
                        const int32_t *seg_adapter, int64_t S, const int64_t *rows,
                        int64_t nrows, double *Y);
void sqo_smoothed_product_rows(const void *X, int dtype, const uint16_t *W, const float *s,
                               int64_t N, int64_t K, const int64_t *rows, int64_t nrows,
                               double *Y);

#ifdef __cplusplus
}
#endif
#endif
