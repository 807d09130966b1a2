/*
 * sage_oracle.h -- declarations of the CPU oracle (test infrastructure only).
 * Layouts are per head, row-major: X[rows, d].  All functions return 0 on
 * success, -1 on bad arguments, -2 on allocation failure.
 */
#ifndef SAGE_ORACLE_H
#define SAGE_ORACLE_H
#include <stdint.h>

float   or_e4m3_decode(uint8_t code);
uint8_t or_e4m3_encode(float x);
float   or_e2m1_decode(uint8_t code);
uint8_t or_e2m1_encode(float x);

int or_mean_rows(const float *X, int64_t rows, int d, float *mean);
int or_block_means(const float *X, int64_t rows, int d, int blk, float *means);
int or_quant_int8(const float *X, int64_t rows, int d, int blk,
                  const float *mean, int mean_per_block, int8_t *out, float *scale);
int or_quant_fp8_per_channel(const float *V, int64_t rows, int d, uint8_t *out, float *scale_v);
int or_delta_s(const float *qbar, int64_t Tm, const float *K, const float *km,
               int64_t N, int d, float *dS);
int or_quant_nvfp4_rows(const float *X, int64_t rows, int d, int blk,
                        const float *mean, int mean_per_block, uint8_t *codes, uint8_t *sf);
int or_quant_nvfp4_cols(const float *V, int64_t rows, int d, uint8_t *codes, uint8_t *sf);
int or_attn_core(const double *Qv, const double *Kv, const double *Vv,
                 const double *row_scale, const double *col_scale,
                 const float *dS, int bq, const double *out_scale,
                 int64_t N, int d, int tile, int causal, double sm_scale,
                 int p_mode, int round32, int64_t r0, int64_t r1, double *out,
                 double *lse /* NULL, or r1 - r0 log-sum-exps of the rows' scores */);
int or_attn_naive_f64(const double *Q, const double *K, const double *V,
                      int64_t N, int d, int causal, double sm_scale,
                      int64_t r0, int64_t r1, double *out);
#endif
