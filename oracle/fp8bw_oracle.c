/*
 * fp8bw_oracle.c -- plain, slow CPU oracle for the blockwise-FP8 linear layer.
 *
 * TEST INFRASTRUCTURE.  Only the test suite, the smoke check and the CPU-baseline
 * leg of the benchmark may call it.  It shares no code, header, table or constant
 * generator with the CUDA library, and neither side includes the other.
 *
 * Source of each definition: Puro-2B ("Poor Lab's Qwen2-1.5B Trained on RTX 5090
 * within $5090", part 3/7), section 3.2 "FP8 Mixed-Precision Training", and the
 * E4M3 format definition of Micikevicius et al. 2022 that section cites.  Points
 * the page leaves open are resolved as follows (plainest reading):
 *   - the scale is FP32 amax/448, one IEEE binary32 division (not amax*(1/448));
 *   - each value is divided by the scale (one binary32 division, round to nearest)
 *     and the FP32 quotient is rounded to E4M3 with ties-to-even, saturating at
 *     +-448: two roundings by definition;
 *   - an all-zero group gets scale 0 and codes 0x00, with no division;
 *   - in a nonzero group the sign of a zero or underflowing value is kept;
 *   - a token count that is not a multiple of 128 leaves a last group of M mod 128
 *     tokens along the token dimension: its amax, and so its scale, is taken over
 *     the tokens present, and codes exist only for them (the same result as
 *     zero-padding the tokens to a multiple of 128, since zeros change no amax).
 *
 * Compile with IEEE binary32 arithmetic (x86-64 SSE, -ffp-contract=off, no
 * fast-math) so that the two divisions round exactly once each.
 */
#include "fp8bw_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ---------------------------------------------------------------- E4M3 ---- */

/* E4M3: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits.  Exponent field 0
 * holds subnormals m/8 * 2^-6; S.1111.111 is NaN; there are no infinities, so the
 * largest finite magnitude is 1.75 * 2^8 = 448. */
double fp8o_e4m3_decode(uint8_t code)
{
    int sign = code >> 7;
    int e = (code >> 3) & 0xF;
    int m = code & 0x7;
    double mag;
    if (e == 0xF && m == 0x7)
        return NAN;
    if (e == 0)
        mag = ldexp((double)m / 8.0, -6);
    else
        mag = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -mag : mag;
}

uint8_t fp8o_e4m3_encode(float v)
{
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs((double)v);
    if (isnan(v))
        return 0x7F;
    if (a >= 448.0)
        return (uint8_t)(sign | 0x7E); /* saturate (ties at 464 also go to 448) */

    /* Spacing of E4M3 values around a: 2^(E-3) in the binade [2^E, 2^(E+1)),
     * E >= -6; the subnormal range below 2^-6 has the spacing of E = -6. */
    int fe;
    frexp(a, &fe);                 /* a = f * 2^fe, f in [0.5, 1) */
    int E = (a == 0.0) ? -6 : fe - 1;
    if (E < -6)
        E = -6;
    double quantum = ldexp(1.0, E - 3);
    double n = a / quantum;        /* exact: division by a power of two */
    double fl = floor(n);
    double frac = n - fl;
    if (frac > 0.5 || (frac == 0.5 && fmod(fl, 2.0) == 1.0))
        fl += 1.0;                 /* round half to even */
    double r = fl * quantum;       /* rounded magnitude, <= 448 */

    if (r == 0.0)
        return sign;
    frexp(r, &fe);
    int E2 = fe - 1;
    if (E2 < -6)                   /* subnormal: r = m * 2^-9 */
        return (uint8_t)(sign | (int)(r / ldexp(1.0, -9)));
    int efield = E2 + 7;
    int mfield = (int)((r / ldexp(1.0, E2) - 1.0) * 8.0);
    return (uint8_t)(sign | (efield << 3) | mfield);
}

void fp8o_e4m3_encode_array(const float *v, int64_t n, uint8_t *out)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i)
        out[i] = fp8o_e4m3_encode(v[i]);
}

/* ------------------------------------------------------------ grouping ---- */

static float bf16_to_float(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

float fp8o_quantize_group(const uint16_t *x, int64_t xstride, int64_t n,
                          uint8_t *q, int64_t qstride)
{
    float amax = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
        float a = fabsf(bf16_to_float(x[i * xstride]));
        if (a > amax)
            amax = a;
    }
    if (amax == 0.0f) {
        for (int64_t i = 0; i < n; ++i)
            q[i * qstride] = 0x00;
        return 0.0f;
    }
    volatile float s = amax / 448.0f;  /* one binary32 division */
    for (int64_t i = 0; i < n; ++i) {
        volatile float quot = bf16_to_float(x[i * xstride]) / s;
        q[i * qstride] = fp8o_e4m3_encode(quot);
    }
    return s;
}

static int bad_sizes(int64_t a, int64_t b)
{
    return a <= 0 || b <= 0 || (a % 128) != 0 || (b % 128) != 0;
}

/* Activations: any token count M > 0, features K a multiple of 128. */
static int bad_act_sizes(int64_t M, int64_t K)
{
    return M <= 0 || K <= 0 || (K % 128) != 0;
}

int fp8o_quant_act(const uint16_t *x, int64_t M, int64_t K, uint8_t *q, float *s)
{
    if (bad_act_sizes(M, K))
        return -1;
    int64_t KB = K / 128;
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t kb = 0; kb < KB; ++kb)
            s[kb * M + m] = fp8o_quantize_group(x + m * K + kb * 128, 1, 128,
                                                q + m * K + kb * 128, 1);
    return 0;
}

int fp8o_quant_act_t(const uint16_t *x, int64_t M, int64_t K, uint8_t *qt, float *st)
{
    if (bad_act_sizes(M, K))
        return -1;
    int64_t MB = (M + 127) / 128; /* the last group may hold fewer than 128 tokens */
#pragma omp parallel for schedule(static)
    for (int64_t k = 0; k < K; ++k)
        for (int64_t mb = 0; mb < MB; ++mb) {
            int64_t n = M - mb * 128 < 128 ? M - mb * 128 : 128;
            st[mb * K + k] = fp8o_quantize_group(x + mb * 128 * K + k, K, n,
                                                 qt + k * M + mb * 128, 1);
        }
    return 0;
}

int fp8o_quant_weight(const uint16_t *w, int64_t N, int64_t K, uint8_t *q, float *s,
                      uint8_t *qt_or_null)
{
    if (bad_sizes(N, K))
        return -1;
    int64_t NB = N / 128, KB = K / 128;
#pragma omp parallel for schedule(static)
    for (int64_t blk = 0; blk < NB * KB; ++blk) {
        int64_t nb = blk / KB, kb = blk % KB;
        const uint16_t *wb = w + nb * 128 * K + kb * 128;
        float amax = 0.0f;
        for (int64_t i = 0; i < 128; ++i)
            for (int64_t j = 0; j < 128; ++j) {
                float a = fabsf(bf16_to_float(wb[i * K + j]));
                if (a > amax)
                    amax = a;
            }
        float sc = 0.0f;
        if (amax != 0.0f) {
            volatile float t = amax / 448.0f;
            sc = t;
        }
        for (int64_t i = 0; i < 128; ++i)
            for (int64_t j = 0; j < 128; ++j) {
                int64_t n = nb * 128 + i, k = kb * 128 + j;
                uint8_t code = 0x00;
                if (amax != 0.0f) {
                    volatile float quot = bf16_to_float(w[n * K + k]) / sc;
                    code = fp8o_e4m3_encode(quot);
                }
                q[n * K + k] = code;
                if (qt_or_null)
                    qt_or_null[k * N + n] = code;
            }
        s[nb * KB + kb] = sc;
    }
    return 0;
}

/* ------------------------------------------------- power-of-two scales ---- */
/*
 * Section 3.2 of the same page: on the RTX 5090 the recipe's 128-blocks run through
 * Transformer Engine's MXFP8 path, where every block scale is a power of two stored
 * as an 8-bit exponent (E8M0).  Reading taken here: the scale of a group is the
 * smallest power of two 2^e with amax <= 448 * 2^e (no value saturates), e clamped to
 * [-127, 127], the E8M0 code being e + 127; an all-zero group takes e = -127 and
 * codes 0x00.  Dividing by 2^e is exact, so each code is the single round-to-
 * nearest-even of x * 2^-e onto E4M3.
 */

int fp8o_e8m0_exponent(float amax)
{
    if (!(amax > 0.0f))
        return -127;
    int E;
    frexp((double)amax, &E);          /* amax = m * 2^E, m in [0.5, 1) */
    int e = E - 10;                   /* 448 * 2^(E-10) < 2^(E-1) <= amax */
    if (e < -127)
        e = -127;
    while ((double)amax > ldexp(448.0, e))
        ++e;
    return e > 127 ? 127 : e;
}

/* One group with a power-of-two scale: codes at q[i*qstride], returns the E8M0 code. */
uint8_t fp8o_quantize_group_e8m0(const uint16_t *x, int64_t xstride, int64_t n,
                                 uint8_t *q, int64_t qstride)
{
    float amax = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
        float a = fabsf(bf16_to_float(x[i * xstride]));
        if (a > amax)
            amax = a;
    }
    if (amax == 0.0f) {
        for (int64_t i = 0; i < n; ++i)
            q[i * qstride] = 0x00;
        return 0;
    }
    int e = fp8o_e8m0_exponent(amax);
    for (int64_t i = 0; i < n; ++i) {
        double v = ldexp((double)bf16_to_float(x[i * xstride]), -e);  /* exact */
        q[i * qstride] = fp8o_e4m3_encode((float)v);
    }
    return (uint8_t)(e + 127);
}

int fp8o_quant_act_e8m0(const uint16_t *x, int64_t M, int64_t K, uint8_t *q, uint8_t *s)
{
    if (bad_sizes(M, K))
        return -1;
    int64_t KB = K / 128;
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t kb = 0; kb < KB; ++kb)
            s[kb * M + m] = fp8o_quantize_group_e8m0(x + m * K + kb * 128, 1, 128,
                                                     q + m * K + kb * 128, 1);
    return 0;
}

int fp8o_quant_act_t_e8m0(const uint16_t *x, int64_t M, int64_t K, uint8_t *qt, uint8_t *st)
{
    if (bad_sizes(M, K))
        return -1;
    int64_t MB = M / 128;
#pragma omp parallel for schedule(static)
    for (int64_t k = 0; k < K; ++k)
        for (int64_t mb = 0; mb < MB; ++mb)
            st[mb * K + k] = fp8o_quantize_group_e8m0(x + mb * 128 * K + k, K, 128,
                                                      qt + k * M + mb * 128, 1);
    return 0;
}

int fp8o_quant_weight_e8m0(const uint16_t *w, int64_t N, int64_t K, uint8_t *q, uint8_t *s,
                           uint8_t *qt_or_null)
{
    if (bad_sizes(N, K))
        return -1;
    int64_t NB = N / 128, KB = K / 128;
#pragma omp parallel for schedule(static)
    for (int64_t blk = 0; blk < NB * KB; ++blk) {
        int64_t nb = blk / KB, kb = blk % KB;
        const uint16_t *wb = w + nb * 128 * K + kb * 128;
        float amax = 0.0f;
        for (int64_t i = 0; i < 128; ++i)
            for (int64_t j = 0; j < 128; ++j) {
                float a = fabsf(bf16_to_float(wb[i * K + j]));
                if (a > amax)
                    amax = a;
            }
        int e = fp8o_e8m0_exponent(amax);
        for (int64_t i = 0; i < 128; ++i)
            for (int64_t j = 0; j < 128; ++j) {
                int64_t n = nb * 128 + i, k = kb * 128 + j;
                uint8_t code = 0x00;
                if (amax != 0.0f)
                    code = fp8o_e4m3_encode((float)ldexp((double)bf16_to_float(w[n * K + k]), -e));
                q[n * K + k] = code;
                if (qt_or_null)
                    qt_or_null[k * N + n] = code;
            }
        s[nb * KB + kb] = (uint8_t)(amax != 0.0f ? e + 127 : 0);
    }
    return 0;
}

/* ---------------------------------------------------------------- GEMM ---- */

/* Decoded value of every code, filled from fp8o_e4m3_decode before any
 * parallel region reads it. */
static double dec_tab[256];
static int dec_tab_ready = 0;

static void fill_dec_tab(void)
{
    if (dec_tab_ready)
        return;
    for (int c = 0; c < 256; ++c)
        dec_tab[c] = fp8o_e4m3_decode((uint8_t)c);
    dec_tab_ready = 1;
}

/* Dequantized B operand element bhat(n, k) for each mode. */
static double bhat(int mode, const uint8_t *b, const float *sb, int64_t N, int64_t K,
                   int64_t n, int64_t k)
{
    switch (mode) {
    case 0: /* FPROP: b[N][K], sb[N/128][K/128] */
        return dec_tab[b[n * K + k]] * (double)sb[(n / 128) * (K / 128) + k / 128];
    case 1: /* DGRAD: b[K][N] (the weight as stored, read transposed), sb[K/128][N/128] */
        return dec_tab[b[k * N + n]] * (double)sb[(k / 128) * (N / 128) + n / 128];
    default: /* WGRAD: b[N][K], sb[K/128][N] */
        return dec_tab[b[n * K + k]] * (double)sb[(k / 128) * N + n];
    }
}

int fp8o_gemm(int mode, const uint8_t *a, const float *sa, const uint8_t *b,
              const float *sb, int64_t M, int64_t N, int64_t K,
              const int64_t *rows, int64_t nrows, double *y, double *asum,
              int nthreads)
{
    /* Tokens may be any count: M for FPROP/DGRAD (a[M][K], sa[K/128][M]), the
     * reduction K for WGRAD (a[M][K], sa[ceil(K/128)][M], sb[ceil(K/128)][N]; the
     * last block holds K mod 128 tokens).  Feature dimensions are multiples of 128. */
    if (mode < 0 || mode > 2 || M <= 0 || N <= 0 || K <= 0 || (N % 128))
        return -1;
    if (mode == 2 ? (M % 128) != 0 : (K % 128) != 0)
        return -1;
    if (!rows)
        nrows = M;
    for (int64_t i = 0; i < nrows && rows; ++i)
        if (rows[i] < 0 || rows[i] >= M)
            return -1;
    fill_dec_tab();
#ifdef _OPENMP
    if (nthreads <= 0)
        nthreads = omp_get_max_threads();
#else
    nthreads = 1;
#endif
    int failed = 0;
#pragma omp parallel num_threads(nthreads)
    {
        double *ahat = (double *)malloc((size_t)K * sizeof(double));
        if (!ahat) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t i = 0; i < nrows; ++i) {
            if (!ahat)
                continue;
            int64_t m = rows ? rows[i] : i;
            /* ahat(m, k) = code value * sa[k/128][m] */
            for (int64_t k = 0; k < K; ++k)
                ahat[k] = dec_tab[a[m * K + k]] * (double)sa[(k / 128) * M + m];
            for (int64_t n = 0; n < N; ++n) {
                double acc = 0.0, aacc = 0.0;
                for (int64_t k = 0; k < K; ++k) {
                    double p = ahat[k] * bhat(mode, b, sb, N, K, n, k);
                    acc += p;
                    aacc += fabs(p);
                }
                y[i * N + n] = acc;
                if (asum)
                    asum[i * N + n] = aacc;
            }
        }
        free(ahat);
    }
    return failed ? -1 : 0;
}

int fp8o_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
