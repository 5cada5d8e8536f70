/*
 * fp8bw_oracle.h -- CPU oracle for the blockwise-FP8 Transformer linear layer.
 *
 * TEST INFRASTRUCTURE.  Only the test suite, the smoke check and the CPU-baseline
 * leg of the benchmark may call anything declared here.  The product library
 * (libfp8bw.so) shares no code with this file and never links it.
 *
 * What it computes (Puro-2B, "Poor Lab's Qwen2-1.5B Trained on RTX 5090 within
 * $5090", part 3/7, section 3.2 "FP8 Mixed-Precision Training"):
 *   - Transformer linear operands are E4M3 (the FP8 format of Micikevicius et al.,
 *     "FP8 Formats for Deep Learning", 2022, cited there).
 *   - Activations and their gradients carry one scale for every 128 neighbouring
 *     elements in the summed (K) direction; weights one scale per 128x128 tile.
 *   - The scales are computed online from the tensor being quantized.  The block
 *     scale is FP32 absmax/448 with saturating round-to-nearest-even onto E4M3,
 *     the DeepSeek-V3 fine-grained recipe that section 3.2 says it follows.
 *   - The forward, input-gradient and weight-gradient GEMMs each take FP8 operands
 *     and return BF16.
 *
 * Layouts (row-major [rows][cols]):
 *   x, w          : BF16 bit patterns (uint16_t)
 *   1x128 scales  : reduction-block-major, s[kb][row] (rows contiguous)
 *   weight scales : s[N/128][K/128]
 *
 * All sizes must be multiples of 128; functions return 0 on success, -1 on a bad
 * size.  Nothing here allocates memory the caller must free.
 */
#ifndef FP8BW_ORACLE_H
#define FP8BW_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* E4M3 (OCP "E4M3FN") value of one code; NaN for 0x7F / 0xFF. */
double fp8o_e4m3_decode(uint8_t code);

/* Round-to-nearest-even of an FP32 value onto the finite E4M3 values, saturating
 * at +-448.  The sign of zero is kept.  NaN input returns 0x7F (outside contract). */
uint8_t fp8o_e4m3_encode(float v);

/* fp8o_e4m3_encode applied to v[0..n-1]. */
void fp8o_e4m3_encode_array(const float *v, int64_t n, uint8_t *out);

/* Quantize one group of n BF16 values read at x[i*xstride], writing codes at
 * q[i*qstride].  Returns the FP32 scale: amax/448 by one binary32 division, or
 * 0.0f (and all codes 0x00) when every value is zero. */
float fp8o_quantize_group(const uint16_t *x, int64_t xstride, int64_t n,
                          uint8_t *q, int64_t qstride);

/* 1x128 groups along K per row: q[M][K], s[K/128][M]. */
int fp8o_quant_act(const uint16_t *x, int64_t M, int64_t K, uint8_t *q, float *s);

/* 1x128 groups along M per column (token-dim grouping for wgrad):
 * qt[K][M] (the transpose of the codes), st[M/128][K]. */
int fp8o_quant_act_t(const uint16_t *x, int64_t M, int64_t K, uint8_t *qt, float *st);

/* 128x128 blocks: q[N][K], s[N/128][K/128], and optionally qt[K][N] = q^T. */
int fp8o_quant_weight(const uint16_t *w, int64_t N, int64_t K, uint8_t *q, float *s,
                      uint8_t *qt_or_null);

/* Power-of-two (E8M0) scales, the MXFP8 form the same section says the recipe runs
 * on its GPUs: the group scale is the smallest 2^e with amax <= 448 * 2^e, e in
 * [-127, 127], stored as the code e + 127 (0 for an all-zero group, whose codes are
 * 0x00); each value's code is RNE(x * 2^-e) onto E4M3 (no saturation occurs). */
int fp8o_e8m0_exponent(float amax);
uint8_t fp8o_quantize_group_e8m0(const uint16_t *x, int64_t xstride, int64_t n,
                                 uint8_t *q, int64_t qstride);
int fp8o_quant_act_e8m0(const uint16_t *x, int64_t M, int64_t K, uint8_t *q, uint8_t *s);
int fp8o_quant_act_t_e8m0(const uint16_t *x, int64_t M, int64_t K, uint8_t *qt, uint8_t *st);
int fp8o_quant_weight_e8m0(const uint16_t *w, int64_t N, int64_t K, uint8_t *q, uint8_t *s,
                           uint8_t *qt_or_null);

/* Modes of the blockwise GEMM, all producing D[M][N] summed over a reduction of
 * length K with one (a-scale x b-scale) pair per 128-long reduction block:
 *   0 FPROP: a[M][K] sa[K/128][M]; b[N][K] sb[N/128][K/128]      (Y  = X  . W^T)
 *   1 DGRAD: a[M][K] sa[K/128][M]; b[K][N] sb[K/128][N/128]      (dX = dY . W)
 *   2 WGRAD: a[M][K] sa[K/128][M]; b[N][K] sb[K/128][N]          (dW = dY^T . X)
 * For each selected row m (rows[i], or every row when rows == NULL) and every n:
 *   y   [i*N + n] = sum_k ahat(m,k) * bhat(n,k)       in FP64
 *   asum[i*N + n] = sum_k |ahat(m,k) * bhat(n,k)|     (may be NULL)
 * where ahat, bhat are the dequantized operands, code value times FP32 scale.
 * One thread computes each output in a fixed order, so the result does not depend
 * on the thread count (nthreads <= 0: OpenMP default). */
int fp8o_gemm(int mode, const uint8_t *a, const float *sa, const uint8_t *b,
              const float *sb, int64_t M, int64_t N, int64_t K,
              const int64_t *rows, int64_t nrows, double *y, double *asum,
              int nthreads);

/* Threads the OpenMP runtime would use for nthreads <= 0. */
int fp8o_max_threads(void);

#ifdef __cplusplus
}
#endif
#endif
