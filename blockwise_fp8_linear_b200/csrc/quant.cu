// quant.cu -- E4M3 quantizers for the blockwise-FP8 linear layer (sm_100a).
//
// Three layouts (Puro-2B part 3/7, section 3.2): 1x128 groups along the reduction
// dimension for activations / activation gradients, the same groups taken along the
// token dimension for wgrad, and 128x128 blocks for weights.  Each group's scale is
// amax/448 in FP32 (one IEEE division); each value is divided by the scale with the
// quotient rounded to FP32, then rounded to nearest-even onto E4M3 with saturation
// at +-448 (cvt.rn.satfinite).  An all-zero group gets scale 0 and codes 0x00.
//
// All three kernels are HBM-bound streaming kernels: 2 bytes read and 1 + 4/128
// bytes written per element.
#include <cstdint>
#include <cuda_runtime.h>

#include "quant.cuh"

namespace fp8bw {

// Two FP32 values -> two E4M3 codes (RNE, saturating); `lo` lands in the low byte.
__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi)
{
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// Per-group division x / s, correctly rounded to binary32.
//
// Fast path (s in [2^-90, 2^90]): one correctly rounded reciprocal r = RN(1/s) per
// group, then per value q0 = RN(x*r), e = x - q0*s (exact by FMA) and
// q = RN(q0 + e*r).  By Markstein's theorem (P. Markstein, "Computation of elementary
// functions on the IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1), 1990;
// also Muller et al., Handbook of Floating-Point Arithmetic, ch. 4) this is the
// correctly rounded quotient whenever no intermediate underflows; quotients small
// enough for that to matter lie far below half the smallest E4M3 subnormal (2^-10),
// where only the sign survives, and the sign is restored from x.  Outside that
// range of s the group falls back to the compiler's IEEE division.  The test suite
// checks the fast path against IEEE division for every (BF16 amax, BF16 x) pair.
struct GroupDiv {
    float s, r;
    bool fast;
    __device__ __forceinline__ explicit GroupDiv(float scale) : s(scale)
    {
        fast = scale >= 0x1p-90f && scale <= 0x1p90f;
        r = fast ? __frcp_rn(scale) : 0.0f;
    }
};

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Fast-path quotients of a pair of values by per-lane-half scales (r, -r and s given
// as packed pairs): q0 = x*r, d = q0*s - x (one FMA, exact), q = q0 - d*r.  The
// residual is taken as q0*s - x rather than x - q0*s so that zeros keep their sign
// with no fix-up: for x = +-0, q0 = +-0 and d = +0, so q = (-0) + (+-0) = +-0; when
// q0 underflows to a zero, d = -x exactly and q = x*r + q0 carries the sign of x; and
// q0 - d*r cannot cancel exactly to zero for a nonzero q0, because |d*r| is within
// an ulp of |q0 - x/s|, far below |q0|.
__device__ __forceinline__ float2 div2_fast(float2 x, float2 r, float2 neg_r, float2 s)
{
    const float2 q0 = __fmul2_rn(x, r);
    const float2 d = __ffma2_rn(q0, s, make_float2(-x.x, -x.y));
    return __ffma2_rn(d, neg_r, q0);
}

// |bf16| max over two packed words, as packed unsigned 16-bit halves (for
// non-negative BF16 values the integer order is the numeric order).
__device__ __forceinline__ uint32_t absmax2(uint32_t a, uint32_t b)
{
    return __vmaxu2(a & 0x7FFF7FFFu, b & 0x7FFF7FFFu);
}

__device__ __forceinline__ float halves_max_to_float(uint32_t m2)
{
    uint32_t m = max(m2 & 0xFFFFu, m2 >> 16);
    return __uint_as_float(m << 16);
}

// Eight BF16 values of one group (one uint4) -> eight E4M3 codes (one uint2), by the
// fast path (r = RN(1/s)) or by IEEE division.
__device__ __forceinline__ uint2 quant8_fast(uint4 v, float r, float s)
{
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    const float2 r2 = make_float2(r, r), nr2 = make_float2(-r, -r), s2 = make_float2(s, s);
    uint32_t c[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 q = div2_fast(make_float2(bf16lo(w[i]), bf16hi(w[i])), r2, nr2, s2);
        c[i] = cvt_e4m3x2(q.x, q.y);
    }
    return make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
}

__device__ __forceinline__ uint2 quant8_ieee(uint4 v, float s)
{
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t c[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
        c[i] = cvt_e4m3x2(__fdiv_rn(bf16lo(w[i]), s), __fdiv_rn(bf16hi(w[i]), s));
    return make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
}

__device__ __forceinline__ uint2 quant8(uint4 v, const GroupDiv &d)
{
    return d.fast ? quant8_fast(v, d.r, d.s) : quant8_ieee(v, d.s);
}

// Power-of-two (E8M0) scales, the MXFP8 form of the recipe (same section): the group
// scale is the smallest 2^e with amax <= 448 * 2^e, e clamped to [-127, 127] (a zero
// or subnormal amax gives -127), stored as the code e + 127.  amax = m * 2^E with
// m in [1, 2): 448 * 2^(E-8) = 1.75 * 2^E >= amax exactly when m <= 1.75, else one
// more power is needed.  Multiplying by 2^-e is exact, so each value's code is a
// single rounding of x * 2^-e onto E4M3 (never saturating).
__device__ __forceinline__ int e8m0_exponent(float amax)
{
    const uint32_t b = __float_as_uint(amax);
    const int be = int(b >> 23);
    if (be == 0)
        return -127;
    const int e = be - 135 + ((b & 0x7FFFFFu) > 0x600000u ? 1 : 0);
    return e < -127 ? -127 : (e > 126 ? 126 : e);
}

// E8M0 scales are stored in the layout the tensor cores read scale factors in: one
// 512-byte block per 128 rows x 128-deep reduction block, in which the code of row r
// fills bytes 16 (r % 32) + 4 (r / 32) .. +3 (repeated for the four 32-wide K steps).
__device__ __forceinline__ uint32_t sf_block_off(int r) { return uint32_t((r & 31) * 16 + ((r >> 5) & 3) * 4); }

__device__ __forceinline__ uint32_t rep4_code(int e, float amax)
{
    return amax != 0.0f ? uint32_t(e + 127) * 0x01010101u : 0u;
}

// 2^-e as a float (e in [-127, 126]).
__device__ __forceinline__ float pow2_neg(int e)
{
    return __uint_as_float(uint32_t(127 - e) << 23);
}

// Eight BF16 values of one group times the power of two `mul` -> eight E4M3 codes.
__device__ __forceinline__ uint2 quant8_pow2(uint4 v, float mul)
{
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    const float2 m2 = make_float2(mul, mul);
    uint32_t c[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 q = __fmul2_rn(make_float2(bf16lo(w[i]), bf16hi(w[i])), m2);
        c[i] = cvt_e4m3x2(q.x, q.y);
    }
    return make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
}

// ------------------------------------------------------------ fp8_quant_act

// A warp quantizes two consecutive groups at a time (half-warp h takes group
// 2p + h); each lane holds 8 consecutive values (16 bytes).  Groups are enumerated
// in memory order, g = m*(K/128) + kb, so the warps in flight stream through one
// contiguous region of X and Q; the scale of group (m, kb) goes to s[kb][m].
constexpr int QA_THREADS = 256;
constexpr int QA_UNROLL = 4;

__global__ void __launch_bounds__(QA_THREADS)
quant_act_kernel(const uint4 *__restrict__ x, int64_t M, int64_t K, uint2 *__restrict__ q,
                 float *__restrict__ s)
{
    const int64_t npairs = M * (K / 128) / 2;
    const int64_t warp = (int64_t(blockIdx.x) * QA_THREADS + threadIdx.x) >> 5;
    const int64_t nwarps = (int64_t(gridDim.x) * QA_THREADS) >> 5;
    const int lane = threadIdx.x & 31;
    const int half = lane >> 4, sub = lane & 15;

    for (int64_t p0 = warp; p0 < npairs; p0 += nwarps * QA_UNROLL) {
        uint4 v[QA_UNROLL];
        int64_t off[QA_UNROLL];
#pragma unroll
        for (int u = 0; u < QA_UNROLL; ++u) {
            int64_t p = p0 + int64_t(u) * nwarps;
            off[u] = -1;
            if (p < npairs) {
                off[u] = (2 * p + half) * 16 + sub;  // in units of 8 elements
                v[u] = __ldg(x + off[u]);
            }
        }
#pragma unroll
        for (int u = 0; u < QA_UNROLL; ++u) {
            int64_t p = p0 + int64_t(u) * nwarps;
            if (p >= npairs)  // uniform across the warp
                break;
            uint32_t m2 = __vmaxu2(absmax2(v[u].x, v[u].y), absmax2(v[u].z, v[u].w));
#pragma unroll
            for (int o = 8; o >= 1; o >>= 1)
                m2 = __vmaxu2(m2, __shfl_xor_sync(0xffffffffu, m2, o));
            float amax = halves_max_to_float(m2);
            float sc = __fdiv_rn(amax, 448.0f);
            uint2 codes = make_uint2(0u, 0u);
            if (amax != 0.0f)
                codes = quant8(v[u], GroupDiv(sc));
            q[off[u]] = codes;
            if (sub == 0) {
                const int64_t g = 2 * p + half, KB = K / 128;
                int64_t m, kb;
                if (g < INT32_MAX) {  // 32-bit division in the common case
                    const uint32_t g32 = uint32_t(g), kb32 = uint32_t(KB);
                    m = g32 / kb32;
                    kb = g32 - uint32_t(m) * kb32;
                } else {
                    m = g / KB;
                    kb = g - m * KB;
                }
                s[kb * M + m] = sc;
            }
        }
    }
}

// ---------------------------------------------------------- fp8_quant_act_t

// Block tile: 128 rows (one token block mb) x 64 columns.  Warp w holds rows
// 16w .. 16w+15; lane l holds columns 2l and 2l+1 of every one of those rows.
// Column absmax: per lane over its 16 rows, then across the 8 warps in shared
// memory.  Each lane then owns 16 consecutive tokens of two columns, which are 16
// contiguous bytes of the transposed output: one 16-byte store per column.
constexpr int QT_THREADS = 256;

__global__ void __launch_bounds__(QT_THREADS)
quant_act_t_kernel(const uint32_t *__restrict__ x, int64_t M, int64_t K,
                   uint8_t *__restrict__ qt, float *__restrict__ st)
{
    __shared__ uint32_t red[8][32];
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    const int64_t k0 = int64_t(blockIdx.x) * 64;
    const int64_t mb = blockIdx.y;
    const int64_t row0 = mb * 128 + 16 * w;

    uint32_t v[16];
#pragma unroll
    for (int r = 0; r < 16; ++r)
        v[r] = __ldg(x + ((row0 + r) * K + k0) / 2 + l);
    uint32_t m2 = 0;
#pragma unroll
    for (int r = 0; r < 16; r += 2)
        m2 = __vmaxu2(m2, absmax2(v[r], v[r + 1]));
    red[w][l] = m2;
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 8; ++i)
        m2 = __vmaxu2(m2, red[i][l]);

    const float amax_lo = __uint_as_float((m2 & 0xFFFFu) << 16);
    const float amax_hi = __uint_as_float(m2 & 0xFFFF0000u);
    const float s_lo = __fdiv_rn(amax_lo, 448.0f);
    const float s_hi = __fdiv_rn(amax_hi, 448.0f);

    // Lane values: v[r] holds (column 2l, column 2l+1) of row r, whose groups have
    // the scales s_lo and s_hi, so each packed pair divides by a packed scale pair.
    uint32_t clo[4] = {0u, 0u, 0u, 0u}, chi[4] = {0u, 0u, 0u, 0u};
    const GroupDiv dlo(s_lo), dhi(s_hi);
    if (dlo.fast && dhi.fast) {
        const float2 r2 = make_float2(dlo.r, dhi.r), nr2 = make_float2(-dlo.r, -dhi.r);
        const float2 s2 = make_float2(s_lo, s_hi);
#pragma unroll
        for (int r = 0; r < 16; r += 2) {
            const float2 a = div2_fast(make_float2(bf16lo(v[r]), bf16hi(v[r])), r2, nr2, s2);
            const float2 b = div2_fast(make_float2(bf16lo(v[r + 1]), bf16hi(v[r + 1])), r2, nr2, s2);
            clo[r / 4] |= cvt_e4m3x2(a.x, b.x) << (16 * ((r / 2) & 1));
            chi[r / 4] |= cvt_e4m3x2(a.y, b.y) << (16 * ((r / 2) & 1));
        }
    } else {
#pragma unroll
        for (int r = 0; r < 16; r += 2) {
            clo[r / 4] |= cvt_e4m3x2(__fdiv_rn(bf16lo(v[r]), s_lo), __fdiv_rn(bf16lo(v[r + 1]), s_lo))
                          << (16 * ((r / 2) & 1));
            chi[r / 4] |= cvt_e4m3x2(__fdiv_rn(bf16hi(v[r]), s_hi), __fdiv_rn(bf16hi(v[r + 1]), s_hi))
                          << (16 * ((r / 2) & 1));
        }
    }
    if (amax_lo == 0.0f)
        clo[0] = clo[1] = clo[2] = clo[3] = 0u;
    if (amax_hi == 0.0f)
        chi[0] = chi[1] = chi[2] = chi[3] = 0u;
    const int64_t col = k0 + 2 * l;
    *reinterpret_cast<uint4 *>(qt + col * M + row0) = make_uint4(clo[0], clo[1], clo[2], clo[3]);
    *reinterpret_cast<uint4 *>(qt + (col + 1) * M + row0) = make_uint4(chi[0], chi[1], chi[2], chi[3]);
    if (w == 0)
        *reinterpret_cast<float2 *>(st + mb * K + col) = make_float2(s_lo, s_hi);
}

// --------------------------------------------------------- fp8_quant_weight

// One block per 128x128 weight block.  Thread t covers, in each of 8 passes, row
// pass*16 + t/16 and columns (t%16)*8 .. +7.
constexpr int QW_THREADS = 256;

// E8: power-of-two scales, s is [N/128][K/128] blocks of 512 bytes, every byte of
// block (nb, kb) the E8M0 code of that weight block.
template <bool E8>
__global__ void __launch_bounds__(QW_THREADS)
quant_weight_kernel(const uint4 *__restrict__ w, int64_t N, int64_t K, uint2 *__restrict__ q,
                    void *__restrict__ s_out, uint8_t *__restrict__ qt)
{
    __shared__ uint32_t red[8];
    __shared__ uint8_t tile[128][144];  // codes, for the optional transposed copy
    const int t = threadIdx.x;
    const int64_t kb = blockIdx.x, nb = blockIdx.y;
    const int rsub = t >> 4, csub = (t & 15) * 8;

    uint4 v[8];
#pragma unroll
    for (int p = 0; p < 8; ++p) {
        int64_t n = nb * 128 + p * 16 + rsub;
        v[p] = __ldg(w + (n * K + kb * 128 + csub) / 8);
    }
    uint32_t m2 = 0;
#pragma unroll
    for (int p = 0; p < 8; ++p)
        m2 = __vmaxu2(m2, __vmaxu2(absmax2(v[p].x, v[p].y), absmax2(v[p].z, v[p].w)));
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1)
        m2 = __vmaxu2(m2, __shfl_xor_sync(0xffffffffu, m2, o));
    if ((t & 31) == 0)
        red[t >> 5] = m2;
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 8; ++i)
        m2 = __vmaxu2(m2, red[i]);
    const float amax = halves_max_to_float(m2);
    const float sc = E8 ? 0.0f : __fdiv_rn(amax, 448.0f);
    const int e = E8 ? e8m0_exponent(amax) : 0;
    const GroupDiv div(sc);

#pragma unroll
    for (int p = 0; p < 8; ++p) {
        int64_t n = nb * 128 + p * 16 + rsub;
        uint2 c = make_uint2(0u, 0u);
        if (amax != 0.0f)
            c = E8 ? quant8_pow2(v[p], pow2_neg(e)) : quant8(v[p], div);
        q[(n * K + kb * 128 + csub) / 8] = c;
        if (qt)
            *reinterpret_cast<uint2 *>(&tile[p * 16 + rsub][csub]) = c;
    }
    if (E8) {
        if (t < 32) {
            const uint32_t w = rep4_code(e, amax);
            reinterpret_cast<uint4 *>(static_cast<uint8_t *>(s_out) + (nb * (K / 128) + kb) * 512)[t] =
                make_uint4(w, w, w, w);
        }
    } else if (t == 0) {
        static_cast<float *>(s_out)[nb * (K / 128) + kb] = sc;
    }
    if (qt) {
        __syncthreads();
        // qt[k][n]: thread t writes column k = t/2 of the block, 64 rows starting at
        // (t%2)*64, as four 16-byte stores.
        const int kk = t >> 1, n0 = (t & 1) * 64;
        uint8_t *dst = qt + (kb * 128 + kk) * N + nb * 128 + n0;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            uint32_t wv[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int r = n0 + c * 16 + j * 4;
                wv[j] = uint32_t(tile[r][kk]) | (uint32_t(tile[r + 1][kk]) << 8) |
                        (uint32_t(tile[r + 2][kk]) << 16) | (uint32_t(tile[r + 3][kk]) << 24);
            }
            *reinterpret_cast<uint4 *>(dst + c * 16) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
        }
    }
}

// ------------------------------------------------------- tile quantizer (dual)

// One CTA per 128 x 128 tile of X (one reduction block of 128 rows).  Every thread
// first loads its 8 x 16 bytes (rows t/16 + 16p, columns 8*(t%16) .. +7), so a CTA
// has its whole 32 KB tile in flight before any arithmetic.
//   ROWS: 1x128 groups along K (the tile's columns) -> q[M][K], s[K/128][M]; each
//         half-warp holds one row, reduced with a 16-lane shuffle.
//   COLS: 1x128 groups along M (the tile's rows) -> qt[K][M], st[M/128][K]; the tile
//         goes through shared memory, thread t takes column pair t%64 over rows
//         32*(t/64) .. +31 (conflict-free 4-byte reads), the four row quarters meet
//         in shared memory for the column absmax.
// With both, X is read once for the two layouts wgrad and fprop/dgrad need.
constexpr int QD_THREADS = 256;

// E8: power-of-two scales in 512-byte blocks (see sf_block_off): s holds
// [M/128][K/128] blocks (row m of block (m/128, kb)), st holds [K/128][M/128] blocks
// (column k of X is row k % 128 of block (k/128, mb)).
// Four CTAs per SM (at most 64 registers): more tiles' loads in flight per SM.
#ifndef FP8BW_QD_MINB
#define FP8BW_QD_MINB 4
#endif
template <bool ROWS, bool COLS, bool E8 = false>
__global__ void __launch_bounds__(QD_THREADS, FP8BW_QD_MINB)
quant_tile_kernel(const uint4 *__restrict__ x, int64_t M, int64_t K, uint2 *__restrict__ q,
                  void *__restrict__ s_out, uint8_t *__restrict__ qt, void *__restrict__ st_out)
{
    __shared__ uint32_t tile[COLS ? 128 * 64 : 1];
    __shared__ uint32_t red[4][64];
    const int t = threadIdx.x;
    const int64_t kb = blockIdx.x, mb = blockIdx.y;
    const int rsub = t >> 4, sub = t & 15;

    uint4 v[8];
#pragma unroll
    for (int p = 0; p < 8; ++p) {
        const int64_t m = mb * 128 + p * 16 + rsub;
        v[p] = __ldg(x + (m * K + kb * 128) / 8 + sub);
    }
    if (ROWS) {
        // Row groups: half-warp h holds rows 16p + rsub (p < 8), 8 values per lane.
        // Each lane's partial amax for its 8 rows goes through a transposing reduction
        // over the 16 lanes (recursive halving: exchange half of the rows' partials with
        // the lane 8, 4, 2 apart, then combine with the lane 1 apart), after which
        // lanes 2p and 2p + 1 hold the amax of row 16p + rsub.  Each lane then works out
        // the scale of that one group, and the quantizing loop fetches group p's
        // scalars by shuffle: the per-group division and reciprocal run once per lane
        // for all 8 groups instead of once per group.
        uint32_t mx[8];
#pragma unroll
        for (int p = 0; p < 8; ++p)
            mx[p] = __vmaxu2(absmax2(v[p].x, v[p].y), absmax2(v[p].z, v[p].w));
        {
            const bool b = (sub & 8) != 0;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t send = b ? mx[j] : mx[j + 4], keep = b ? mx[j + 4] : mx[j];
                mx[j] = __vmaxu2(keep, __shfl_xor_sync(0xffffffffu, send, 8));
            }
        }
        {
            const bool b = (sub & 4) != 0;
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const uint32_t send = b ? mx[j] : mx[j + 2], keep = b ? mx[j + 2] : mx[j];
                mx[j] = __vmaxu2(keep, __shfl_xor_sync(0xffffffffu, send, 4));
            }
        }
        {
            const bool b = (sub & 2) != 0;
            const uint32_t send = b ? mx[0] : mx[1], keep = b ? mx[1] : mx[0];
            mx[0] = __vmaxu2(keep, __shfl_xor_sync(0xffffffffu, send, 2));
        }
        mx[0] = __vmaxu2(mx[0], __shfl_xor_sync(0xffffffffu, mx[0], 1));
        const float amax = halves_max_to_float(mx[0]);
        const int64_t m_own = mb * 128 + (sub >> 1) * 16 + rsub;
        // per group: E8 the multiplier 2^-e (0 for an all-zero group); FP32 the scale
        // (0 for an all-zero group) and RN(1/s), or -1 when the group takes IEEE division
        float g0 = 0.0f, g1 = 0.0f;
        if constexpr (E8) {
            const int e = e8m0_exponent(amax);
            g0 = amax != 0.0f ? pow2_neg(e) : 0.0f;
            if ((sub & 1) == 0)
                *reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(s_out) +
                                              ((m_own >> 7) * (K / 128) + kb) * 512 +
                                              sf_block_off(int(m_own & 127))) = rep4_code(e, amax);
        } else {
            g0 = __fdiv_rn(amax, 448.0f);
            const GroupDiv d(g0);
            g1 = d.fast ? d.r : -1.0f;
            if ((sub & 1) == 0)
                static_cast<float *>(s_out)[kb * M + m_own] = g0;
        }
#pragma unroll
        for (int p = 0; p < 8; ++p) {
            const int row = p * 16 + rsub;
            const int64_t m = mb * 128 + row;
            const float gp = __shfl_sync(0xffffffffu, g0, 2 * p, 16);
            uint2 codes = make_uint2(0u, 0u);
            if constexpr (E8) {
                if (gp != 0.0f)
                    codes = quant8_pow2(v[p], gp);
            } else {
                const float rp = __shfl_sync(0xffffffffu, g1, 2 * p, 16);
                if (gp != 0.0f)
                    codes = rp > 0.0f ? quant8_fast(v[p], rp, gp) : quant8_ieee(v[p], gp);
            }
            q[(m * K + kb * 128) / 8 + sub] = codes;
            if (COLS)
                *reinterpret_cast<uint4 *>(&tile[row * 64 + sub * 4]) = v[p];
        }
    } else if (COLS) {
#pragma unroll
        for (int p = 0; p < 8; ++p)
            *reinterpret_cast<uint4 *>(&tile[(p * 16 + rsub) * 64 + sub * 4]) = v[p];
    }
    if (COLS) {
        __syncthreads();
        const int cp = t & 63, rq = t >> 6;
        uint32_t w[32];
#pragma unroll
        for (int i = 0; i < 32; ++i)
            w[i] = tile[(rq * 32 + i) * 64 + cp];
        uint32_t m2 = 0;
#pragma unroll
        for (int i = 0; i < 32; i += 2)
            m2 = __vmaxu2(m2, absmax2(w[i], w[i + 1]));
        red[rq][cp] = m2;
        __syncthreads();
        m2 = __vmaxu2(__vmaxu2(red[0][cp], red[1][cp]), __vmaxu2(red[2][cp], red[3][cp]));
        const float amax_lo = __uint_as_float((m2 & 0xFFFFu) << 16);
        const float amax_hi = __uint_as_float(m2 & 0xFFFF0000u);
        const float s_lo = E8 ? 0.0f : __fdiv_rn(amax_lo, 448.0f);
        const float s_hi = E8 ? 0.0f : __fdiv_rn(amax_hi, 448.0f);
        const int e_lo = E8 ? e8m0_exponent(amax_lo) : 0;
        const int e_hi = E8 ? e8m0_exponent(amax_hi) : 0;
        uint32_t clo[8], chi[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
            clo[i] = chi[i] = 0u;
        const GroupDiv dlo(s_lo), dhi(s_hi);
        if (E8) {
            const float2 mul2 = make_float2(pow2_neg(e_lo), pow2_neg(e_hi));
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
                const float2 a = __fmul2_rn(make_float2(bf16lo(w[i]), bf16hi(w[i])), mul2);
                const float2 b = __fmul2_rn(make_float2(bf16lo(w[i + 1]), bf16hi(w[i + 1])), mul2);
                clo[i / 4] |= cvt_e4m3x2(a.x, b.x) << (16 * ((i / 2) & 1));
                chi[i / 4] |= cvt_e4m3x2(a.y, b.y) << (16 * ((i / 2) & 1));
            }
        } else if (dlo.fast && dhi.fast) {
            const float2 r2 = make_float2(dlo.r, dhi.r), nr2 = make_float2(-dlo.r, -dhi.r);
            const float2 s2 = make_float2(s_lo, s_hi);
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
                const float2 a = div2_fast(make_float2(bf16lo(w[i]), bf16hi(w[i])), r2, nr2, s2);
                const float2 b = div2_fast(make_float2(bf16lo(w[i + 1]), bf16hi(w[i + 1])), r2, nr2, s2);
                clo[i / 4] |= cvt_e4m3x2(a.x, b.x) << (16 * ((i / 2) & 1));
                chi[i / 4] |= cvt_e4m3x2(a.y, b.y) << (16 * ((i / 2) & 1));
            }
        } else {
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
                clo[i / 4] |= cvt_e4m3x2(__fdiv_rn(bf16lo(w[i]), s_lo),
                                         __fdiv_rn(bf16lo(w[i + 1]), s_lo))
                              << (16 * ((i / 2) & 1));
                chi[i / 4] |= cvt_e4m3x2(__fdiv_rn(bf16hi(w[i]), s_hi),
                                         __fdiv_rn(bf16hi(w[i + 1]), s_hi))
                              << (16 * ((i / 2) & 1));
            }
        }
        if (amax_lo == 0.0f) {
#pragma unroll
            for (int i = 0; i < 8; ++i)
                clo[i] = 0u;
        }
        if (amax_hi == 0.0f) {
#pragma unroll
            for (int i = 0; i < 8; ++i)
                chi[i] = 0u;
        }
        const int64_t col = kb * 128 + 2 * cp;
        const int64_t m0 = mb * 128 + rq * 32;
        uint4 *dlo_p = reinterpret_cast<uint4 *>(qt + col * M + m0);
        uint4 *dhi_p = reinterpret_cast<uint4 *>(qt + (col + 1) * M + m0);
        dlo_p[0] = make_uint4(clo[0], clo[1], clo[2], clo[3]);
        dlo_p[1] = make_uint4(clo[4], clo[5], clo[6], clo[7]);
        dhi_p[0] = make_uint4(chi[0], chi[1], chi[2], chi[3]);
        dhi_p[1] = make_uint4(chi[4], chi[5], chi[6], chi[7]);
        if (rq == 0) {
            if (E8) {
                uint8_t *blk = static_cast<uint8_t *>(st_out) + ((col >> 7) * (M / 128) + mb) * 512;
                *reinterpret_cast<uint32_t *>(blk + sf_block_off(int(col & 127))) = rep4_code(e_lo, amax_lo);
                *reinterpret_cast<uint32_t *>(blk + sf_block_off(int((col + 1) & 127))) = rep4_code(e_hi, amax_hi);
            } else
                *reinterpret_cast<float2 *>(static_cast<float *>(st_out) + mb * K + col) =
                    make_float2(s_lo, s_hi);
        }
    }
}

// ------------------------------------------------------------------ launchers

#ifndef FP8BW_QUANT_TILE
#define FP8BW_QUANT_TILE 1
#endif

cudaError_t launch_quant_act(const void *x, int64_t M, int64_t K, uint8_t *q, float *s,
                             cudaStream_t stream, int num_sms)
{
    if (FP8BW_QUANT_TILE) {
        dim3 grid(unsigned(K / 128), unsigned(M / 128));
        quant_tile_kernel<true, false><<<grid, QD_THREADS, 0, stream>>>(
            static_cast<const uint4 *>(x), M, K, reinterpret_cast<uint2 *>(q), s, nullptr,
            nullptr);
        return cudaGetLastError();
    }
    const int64_t npairs = M * (K / 128) / 2;
    const int64_t warps_needed = (npairs + QA_UNROLL - 1) / QA_UNROLL;
    int64_t blocks = (warps_needed + (QA_THREADS / 32) - 1) / (QA_THREADS / 32);
    const int64_t cap = int64_t(num_sms) * 8;
    if (blocks > cap)
        blocks = cap;
    quant_act_kernel<<<dim3(unsigned(blocks)), QA_THREADS, 0, stream>>>(
        static_cast<const uint4 *>(x), M, K, reinterpret_cast<uint2 *>(q), s);
    return cudaGetLastError();
}

cudaError_t launch_quant_dual(const void *x, int64_t M, int64_t K, uint8_t *q, float *s,
                              uint8_t *qt, float *st, cudaStream_t stream)
{
    dim3 grid(unsigned(K / 128), unsigned(M / 128));
    quant_tile_kernel<true, true><<<grid, QD_THREADS, 0, stream>>>(
        static_cast<const uint4 *>(x), M, K, reinterpret_cast<uint2 *>(q), s, qt, st);
    return cudaGetLastError();
}

cudaError_t launch_quant_act_t(const void *x, int64_t M, int64_t K, uint8_t *qt, float *st,
                               cudaStream_t stream)
{
    if (FP8BW_QUANT_TILE) {
        dim3 grid(unsigned(K / 128), unsigned(M / 128));
        quant_tile_kernel<false, true><<<grid, QD_THREADS, 0, stream>>>(
            static_cast<const uint4 *>(x), M, K, nullptr, nullptr, qt, st);
        return cudaGetLastError();
    }
    dim3 grid(unsigned(K / 64), unsigned(M / 128));
    quant_act_t_kernel<<<grid, QT_THREADS, 0, stream>>>(static_cast<const uint32_t *>(x), M, K,
                                                       qt, st);
    return cudaGetLastError();
}

cudaError_t launch_quant_weight(const void *w, int64_t N, int64_t K, uint8_t *q, float *s,
                                uint8_t *qt, cudaStream_t stream)
{
    dim3 grid(unsigned(K / 128), unsigned(N / 128));
    quant_weight_kernel<false><<<grid, QW_THREADS, 0, stream>>>(
        static_cast<const uint4 *>(w), N, K, reinterpret_cast<uint2 *>(q), s, qt);
    return cudaGetLastError();
}

// Power-of-two (E8M0) scale quantizers: the same code layouts, scales as 512-byte
// tensor-core scale blocks.
cudaError_t launch_quant_e8m0(int which, const void *x, int64_t M, int64_t K, uint8_t *q,
                              uint8_t *s, uint8_t *qt, uint8_t *st, cudaStream_t stream)
{
    dim3 grid(unsigned(K / 128), unsigned(M / 128));
    const uint4 *xv = static_cast<const uint4 *>(x);
    uint2 *qv = reinterpret_cast<uint2 *>(q);
    switch (which) {
    case 0:  // rows: q[M][K], s[K/128][M]
        quant_tile_kernel<true, false, true><<<grid, QD_THREADS, 0, stream>>>(xv, M, K, qv, s,
                                                                            nullptr, nullptr);
        break;
    case 1:  // token groups: qt[K][M], st[M/128][K]
        quant_tile_kernel<false, true, true><<<grid, QD_THREADS, 0, stream>>>(xv, M, K, nullptr,
                                                                            nullptr, qt, st);
        break;
    case 2:  // both
        quant_tile_kernel<true, true, true><<<grid, QD_THREADS, 0, stream>>>(xv, M, K, qv, s, qt,
                                                                           st);
        break;
    default:  // weight blocks: q[N=M][K], s[M/128][K/128], optional qt[K][M]
        quant_weight_kernel<true><<<grid, QW_THREADS, 0, stream>>>(xv, M, K, qv, s, qt);
        break;
    }
    return cudaGetLastError();
}

} // namespace fp8bw
