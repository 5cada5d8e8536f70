/*
 * fp8bw.h -- C ABI of the blockwise-FP8 Transformer linear layer for NVIDIA B200
 * (sm_100a).
 *
 * The operations follow Puro-2B ("Poor Lab's Qwen2-1.5B Trained on RTX 5090 within
 * $5090", arXiv HTML part 3/7), section 3.2 "FP8 Mixed-Precision Training":
 * Transformer linear layers quantize their BF16 inputs and weights to E4M3
 * immediately before each GEMM.  Activations and their gradients carry a scale for
 * every 128 neighbouring elements in the direction the GEMM sums over, weights a
 * scale for every 128x128 tile; fprop, dgrad and wgrad all run in FP8 and the layer
 * hands a BF16 result back to the model.  Each block scale is the block's absolute
 * maximum divided by 448 (the largest finite E4M3 magnitude) in FP32, and values are
 * divided by it and rounded to nearest-even onto E4M3, saturating at +-448 (the
 * fine-grained recipe section 3.2 says it follows, DeepSeek-V3).
 *
 * Conventions for every entry point
 *   Pointers     Device (or managed) pointers on the calling thread's current CUDA
 *                device, unless stated otherwise; a host pointer or a buffer of
 *                another device returns FP8BW_EINVAL before anything is launched.
 *                The library never changes the current device.  The caller
 *                allocates and owns every buffer; the library never frees caller
 *                memory and keeps no pointer after the call returns.
 *   Layouts      Row-major [rows][cols].  BF16 tensors are IEEE bfloat16.  FP8 codes
 *                are E4M3 ("E4M3FN": bias 7, no infinities, NaN = S.1111.111).
 *                1x128 scale tensors are reduction-block-major, s[kb][row], so one
 *                tile's scales for one reduction block are contiguous.
 *   Sizes        Every dimension must be a positive multiple of 128 and at most
 *                FP8BW_MAX_DIM (else FP8BW_ESHAPE), except a token count: the M of
 *                fp8_quant_act, fp8_quant_act_t, fp8_quant_act_dual and of the FPROP
 *                and DGRAD GEMMs, and the reduction K of the WGRAD GEMM and of
 *                fp8_gemm_wgrad_acc32, which need only be a positive multiple of 16
 *                (the 16-byte row stride of token-major codes).  The last group of
 *                128 tokens may then be partial: its amax and scale are taken over
 *                the tokens present (the result of zero-padding the tokens to a
 *                multiple of 128, restricted to the tokens present), so token-wise
 *                scale arrays have ceil(tokens/128) rows.  The E8M0 entry points
 *                keep whole groups.
 *   Alignment    Every pointer must be 16-byte aligned (else FP8BW_EALIGN).
 *   Streams      `stream` is a cudaStream_t (NULL = legacy default stream).  Work is
 *                enqueued asynchronously; no call but fp8bw_last_device_error
 *                synchronizes the stream.  Calls on distinct streams may run
 *                concurrently from different threads.  A call only enqueues
 *                kernels (it allocates nothing and waits for
 *                nothing), so it may be captured into a CUDA graph once its
 *                configuration has run eagerly on the device (the first launch of a
 *                configuration sets its shared-memory limit); fp8bw_last_device_error
 *                must stay outside a capture.
 *   Errors       Every call returns an fp8bw_status and never aborts or throws.
 *                Argument errors are reported before anything is launched.  A failed
 *                launch returns FP8BW_ECUDA.  The GEMMs and the activation quantizers
 *                bound every wait inside their kernels; a wait that runs out sets a
 *                per-device error word that fp8bw_last_device_error() reads.
 *   Inputs       Finite BF16 values.  Non-finite inputs give unspecified codes but
 *                never fault.
 *   Memory       The library allocates no device memory: the per-device error words
 *                are static device variables and TMA descriptors are passed by value.
 */
#ifndef FP8BW_H
#define FP8BW_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FP8BW_OK = 0,
    FP8BW_EINVAL = 1,      /* null pointer or bad mode */
    FP8BW_EALIGN = 2,      /* a pointer is not 16-byte aligned */
    FP8BW_ESHAPE = 3,      /* a size is not a positive multiple of 128 (16 for a token count), or too large */
    FP8BW_ECUDA = 4,       /* a CUDA runtime call or kernel launch failed */
    FP8BW_ETIMEOUT = 5,    /* a bounded in-kernel wait ran out (from fp8bw_last_device_error) */
    FP8BW_EUNSUPPORTED = 6 /* the current device is not sm_100 */
} fp8bw_status;

typedef enum { FP8BW_FPROP = 0, FP8BW_DGRAD = 1, FP8BW_WGRAD = 2 } fp8bw_mode;

#define FP8BW_MAX_DIM (1 << 20)

/*
 * fp8_quant_act -- 1x128 groups along the reduction dimension (section 3.2: the
 * scales of activations and of their gradients are taken over runs of 128 adjacent
 * elements in the direction the GEMM sums over).
 *   x  [M][K] BF16 in      q [M][K] E4M3 codes out      s [K/128][M] FP32 out
 * For each row m and block kb: amax = max |x[m][kb*128 .. kb*128+127]|,
 * s[kb][m] = amax / 448 (binary32 division), q = e4m3_rne_sat(x / s) with the
 * quotient rounded to binary32 first.  An all-zero group gets s = 0 and codes 0x00.
 * Used for X before fprop (K = in_features) and dY before dgrad (K = out_features).
 */
int fp8_quant_act(const void *x_bf16, int64_t M, int64_t K, uint8_t *q, float *s,
                  void *stream);

/*
 * fp8_quant_act_t -- the same groups taken along M (the token dimension), the
 * grouping wgrad needs because its reduction runs over tokens (section 3.2: wgrad
 * runs in FP8 on the layer's inputs and output gradients).
 *   x  [M][K] BF16 in      qt [K][M] E4M3 codes out (transposed)      st [ceil(M/128)][K] FP32 out
 * For each column k and block mb: the group is x[mb*128 .. mb*128+127][k];
 * st[mb][k] is its scale and qt[k][mb*128 + i] its codes.  Quantized from the BF16
 * tensor, not from the row-wise FP8 copy.
 */
int fp8_quant_act_t(const void *x_bf16, int64_t M, int64_t K, uint8_t *qt, float *st,
                    void *stream);

/*
 * fp8_quant_act_dual -- both activation layouts from one read of X (section 3.2:
 * wgrad reuses the FP8 copy of the layer input made for fprop; this call produces,
 * in one pass over the BF16 tensor, the row-wise copy fprop/dgrad consume and the
 * token-wise copy wgrad consumes).  Outputs are bit-identical to fp8_quant_act(x, M, K, q, s) and
 * fp8_quant_act_t(x, M, K, qt, st):
 *   x [M][K] BF16 in
 *   q [M][K], s [K/128][M]      1x128 groups along K
 *   qt [K][M], st [ceil(M/128)][K]    1x128 groups along M (codes transposed)
 */
int fp8_quant_act_dual(const void *x_bf16, int64_t M, int64_t K, uint8_t *q, float *s,
                       uint8_t *qt, float *st, void *stream);

/*
 * fp8_quant_weight -- 128x128 blocks (section 3.2: a weight's scales are taken
 * over square 128x128 tiles).
 *   w  [N][K] BF16 in      q [N][K] E4M3 out      s [N/128][K/128] FP32 out
 *   qt_or_null: if not NULL, also writes qt [K][N] = q transposed (same codes; a
 *   128x128 block keeps its one scale under transposition).
 */
int fp8_quant_weight(const void *w_bf16, int64_t N, int64_t K, uint8_t *q, float *s,
                     uint8_t *qt_or_null, void *stream);

/*
 * fp8_gemm_blockwise -- D[M][N] (BF16) = sum over a reduction of length K, with the
 * reduction cut into 128-long blocks kb.  For each kb the FP8 partial product
 * sum_{k in kb} qa*qb is accumulated in FP32 by the tensor cores and then promoted
 * into an FP32 running sum multiplied by (a-scale x b-scale) of that block; the sum
 * is rounded to BF16 (nearest-even) at the end.  Section 3.2: the forward, input-gradient
 * and weight-gradient GEMMs of these layers all run in FP8, and the model receives
 * BF16 results.
 *
 *   FPROP  Y  = X . W^T   a = Qx  [M][K], sa = [K/128][M]   (from fp8_quant_act(X))
 *                         b = Qw  [N][K], sb = [N/128][K/128] (from fp8_quant_weight(W))
 *                         M = tokens, K = in_features, N = out_features
 *   DGRAD  dX = dY . W    a = Qdy [M][K], sa = [K/128][M]   (from fp8_quant_act(dY))
 *                         b = Qw  [K][N], sb = [K/128][N/128] (the weight exactly as
 *                         fp8_quant_weight produced it, [out][in]; read transposed)
 *                         M = tokens, K = out_features, N = in_features
 *   WGRAD  dW = dY^T . X  a = Qdy^T [M][K], sa = [K/128][M] (from fp8_quant_act_t(dY))
 *                         b = Qx^T  [N][K], sb = [K/128][N] (from fp8_quant_act_t(X));
 *                         with K tokens not a multiple of 128, sa and sb have
 *                         ceil(K/128) rows, the last for the partial token group
 *                         M = out_features, K = tokens, N = in_features
 * d_bf16 [M][N] is written, never read.
 */
int fp8_gemm_blockwise(int mode, const uint8_t *a, const float *sa, const uint8_t *b,
                       const float *sb, void *d_bf16, int64_t M, int64_t N, int64_t K,
                       void *stream);

/*
 * fp8_gemm_wgrad_acc32 -- wgrad with FP32 gradient accumulation (the reading notes on
 * the same paper, section 2.3: gradient accumulation stays in FP32).  Same operands
 * and promotion as fp8_gemm_blockwise(FP8BW_WGRAD, ...), but the FP32 running sum is
 * added into dw32 instead of being rounded to BF16:
 *   dw32 [M][N] FP32, read and written: dw32 += sum over the token blocks
 * (M = out_features, N = in_features, K = tokens).  Calls that overlap on the GPU and
 * target the same dw32 may interleave their additions (the sum is the same up to
 * FP32 rounding order).
 */
int fp8_gemm_wgrad_acc32(const uint8_t *a, const float *sa, const uint8_t *b, const float *sb,
                         float *dw32, int64_t M, int64_t N, int64_t K, void *stream);

/*
 * ---- Power-of-two (E8M0) scales: the MXFP8 form of the recipe ----
 * Section 3.2: on the RTX 5090 the 128-blocks run through Transformer Engine's MXFP8
 * path, where every block scale is a power of two stored as an 8-bit exponent.
 * These entry points keep the groupings and code layouts above; each scale is the
 * E8M0 code e + 127 of 2^e, the smallest power of two with amax <= 448 * 2^e (e
 * clamped to [-127, 127]), and each value's code is the round-to-nearest-even of
 * x * 2^-e onto E4M3, which never saturates.  An all-zero group gets code 0 and
 * codes 0x00.
 *
 * Scale layout (the one the tensor cores read scale factors in): 512-byte blocks, one
 * per 128 rows x 128-deep reduction block; in a block the code of row r (0..127)
 * fills bytes 16 (r % 32) + 4 (r / 32) .. +3 (the code repeated four times, once per
 * 32-wide K step of the MMA).
 *   fp8_quant_act_e8m0       x[M][K] -> q[M][K]; s: [M/128][K/128] blocks, rows m
 *   fp8_quant_act_t_e8m0     x[M][K] -> qt[K][M]; st: [K/128][M/128] blocks, the
 *                            columns k of x as rows (the wgrad operand's rows)
 *   fp8_quant_act_dual_e8m0  both, from one read of x
 *   fp8_quant_weight_e8m0    w[N][K] -> q[N][K]; s: [N/128][K/128] blocks, every byte
 *                            of block (nb, kb) the code of that weight block;
 *                            optional qt[K][N]
 * Buffer sizes: M*K/32 bytes of scales for the activation forms, N*K/32 for the
 * weight.  Errors and pointer rules as above (every pointer 16-byte aligned).
 */
int fp8_quant_act_e8m0(const void *x_bf16, int64_t M, int64_t K, uint8_t *q, uint8_t *s_e8m0,
                       void *stream);
int fp8_quant_act_t_e8m0(const void *x_bf16, int64_t M, int64_t K, uint8_t *qt,
                         uint8_t *st_e8m0, void *stream);
int fp8_quant_act_dual_e8m0(const void *x_bf16, int64_t M, int64_t K, uint8_t *q,
                            uint8_t *s_e8m0, uint8_t *qt, uint8_t *st_e8m0, void *stream);
int fp8_quant_weight_e8m0(const void *w_bf16, int64_t N, int64_t K, uint8_t *q,
                          uint8_t *s_e8m0, uint8_t *qt_or_null, void *stream);

/*
 * fp8_gemm_blockwise_e8m0 -- fp8_gemm_blockwise with E8M0 scales (same modes and
 * operand layouts; sa / sb the scale blocks above: FPROP sa from fp8_quant_act_e8m0,
 * sb from fp8_quant_weight_e8m0; DGRAD the same weight blocks, read transposed;
 * WGRAD both from fp8_quant_act_t_e8m0).  The scales are applied
 * by the tensor cores (tcgen05.mma kind::mxf8f6f4.block_scale, each 128-block's
 * scale repeated over its four 32-wide K steps), so the reduction accumulates in one
 * FP32 accumulator and the result is rounded to BF16 once: D = sum_k
 * (qa 2^ea)(qb 2^eb).  d_bf16 [M][N] is written, never read.
 */
int fp8_gemm_blockwise_e8m0(int mode, const uint8_t *a, const uint8_t *sa_e8m0,
                            const uint8_t *b, const uint8_t *sb_e8m0, void *d_bf16, int64_t M,
                            int64_t N, int64_t K, void *stream);

/* Human-readable name of a status code (static string). */
const char *fp8bw_status_string(int status);

/* Synchronizes `stream`, then reads and clears the current device's error word:
 * FP8BW_OK, or FP8BW_ETIMEOUT if a bounded in-kernel wait ran out since the last
 * call (the GEMM or quantizer whose wait ran out returned early and its output is
 * undefined). */
int fp8bw_last_device_error(void *stream);

/* Self-test of the failure-detection path (no counterpart in the paper; it checks
 * this library's own bounded waits).  Launches one warp on `stream` that waits, with
 * the GEMM's bounded wait, on a barrier nothing arrives on; after limit_us
 * microseconds (1 .. 1e6, else FP8BW_EINVAL) the wait gives up, records a timeout in
 * the device error word and the kernel returns.  fp8bw_last_device_error() then
 * reports FP8BW_ETIMEOUT once; the device stays usable. */
int fp8bw_selftest_wait_timeout(int64_t limit_us, void *stream);

/* Library version, e.g. "fp8bw 0.1 sm_100a". */
const char *fp8bw_version(void);

#ifdef __cplusplus
}
#endif
#endif /* FP8BW_H */
