/*
 * fp4_oracle.h -- C interface of the CPU oracle (test infrastructure only;
 * see fp4_oracle.c for the readings it follows).  All pointers are host
 * pointers; bf16 and fp16 values are passed as raw uint16 bit patterns.
 */
#ifndef FP4_ORACLE_H
#define FP4_ORACLE_H
#include <stdint.h>

#define ORC_SCALE_F32 0
#define ORC_SCALE_F16 1

#define ORC_OK 0
#define ORC_ERR_ARG 1
#define ORC_ERR_NONFINITE 2
#define ORC_ERR_SCALE 3
#define ORC_ERR_ALLOC 4

int orc_format_bias(int fmt);
double orc_code_value(int fmt, int code);
void orc_format_table(int fmt, double mags[8], double *qmax);
float orc_bias_factor(int j);
uint16_t orc_f32_to_bf16(float f);
float orc_bf16_to_f32(uint16_t h);
uint16_t orc_f32_to_f16(float f);
float orc_f16_to_f32(uint16_t h);
int orc_nearest_index(double a, const double mags[8]);
int orc_quantize_fixed(const float *W, int N, int K, int g, int fmt, int j, const int8_t *shift,
                       int sdt, uint8_t *packed, void *scales, double *sse_out);
int orc_quantize(const float *W, int N, int K, int g, int fmt_mode, int bias_search,
                 const int8_t *shift, int sdt, uint8_t *packed, void *scales, int32_t choice[2],
                 double sse24[24]);
int orc_dequantize(const uint8_t *packed, const void *scales, int sdt, int fmt, int N, int K, int g,
                   double *W_hat);
int orc_gemm(const uint16_t *X, const uint8_t *packed, const void *scales, int sdt, int fmt, int M,
             int N, int K, int g, float rho, double *Y);
int orc_gemm_sampled(const uint16_t *X, const uint8_t *packed, const void *scales, int sdt, int fmt,
                     int M, int N, int K, int g, float rho, int count, const int32_t *ms,
                     const int32_t *ns, double *out);
int orc_preshift_calibrate(const uint16_t *X, int M, int K, int8_t *shift, float *rho_out);
int orc_preshift_apply(const uint16_t *X, int M, int K, const int8_t *shift, float rho, uint16_t *Xt);
/* granularity of the scale (reading R11) */
#define ORC_GRAN_GROUP 0   /* g consecutive elements of a row */
#define ORC_GRAN_CHANNEL 1 /* one output channel: a whole row */
#define ORC_GRAN_HEAD 2    /* N/heads consecutive rows (one attention head) */
int orc_block_count(int N, int K, int g, int gran, int heads);
int orc_quantize_blocks(const float *W, int N, int K, int g, int gran, int heads, int fmt, int j,
                        const int8_t *jforce, const int8_t *shift, int sdt, uint8_t *packed,
                        void *scales, int8_t *jmap, double *sse_out);
/* 4-bit activations with the pre-shifted bias (reading R10) */
int orc_act_quantize(const uint16_t *X, int M, int K, const int8_t *shift, float rho, int fmt, int j,
                     uint8_t *packed, float *s_out);
int orc_gemm_w4a4(const uint8_t *apacked, int afmt, float s_a, const uint8_t *packed,
                  const void *scales, int sdt, int fmt, int M, int N, int K, int g, double *Y);
int orc_gemm_w4a4_sampled(const uint8_t *apacked, int afmt, float s_a, const uint8_t *packed,
                          const void *scales, int sdt, int fmt, int M, int N, int K, int g,
                          int count, const int32_t *ms, const int32_t *ns, double *out);
int orc_num_threads(void);
void orc_set_num_threads(int n);

#endif
