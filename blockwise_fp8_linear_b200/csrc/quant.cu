// quant.cu -- E4M3 quantizers for the blockwise-FP8 linear layer (sm_100a).
//
// Three layouts (Puro-2B part 3/7, section 3.2): 1x128 groups along the reduction
// dimension for activations / activation gradients, the same groups taken along the
// token dimension for wgrad, and 128x128 blocks for weights.  Each group's scale is
// amax/448 in FP32 (one IEEE division); each value is divided by the scale with the
// quotient rounded to FP32, then rounded to nearest-even onto E4M3 with saturation
// at +-448 (cvt.rn.satfinite).  An all-zero group gets scale 0 and codes 0x00.
//
// Both kernels (the tile quantizer for activations, the block quantizer for weights)
// are HBM-bound streaming kernels: 2 bytes read and 1 + 4/128 bytes written per
// element and layout.
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "launch_cache.cuh"
#include "ptx.cuh"
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

// The group scale amax / 448, correctly rounded to binary32, in three operations
// instead of a full division: q0 = RN(amax * RN(1/448)), then one correction step
// (Markstein's, as in GroupDiv below): d = RN(amax - q0 * 448) by FMA, s = RN(q0 + d *
// RN(1/448)).  amax is always a non-negative BF16 value widened to FP32 (32,640
// positive finite ones and zero); the sequence equals the IEEE quotient for every one
// of them, checked against the exact rational quotient on the host and against the
// oracle on the GPU for every BF16 amax.
__device__ __forceinline__ float scale_of_amax(float amax)
{
    constexpr float inv448 = 1.0f / 448.0f;
    const float q0 = __fmul_rn(amax, inv448);
    const float d = __fmaf_rn(-q0, 448.0f, amax);
    return __fmaf_rn(d, inv448, q0);
}

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
    pdl_wait();
    pdl_launch_dependents();

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
    const float sc = E8 ? 0.0f : scale_of_amax(amax);
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

// ------------------------------------------------------------ tile quantizer

// One CTA per 128 x 128 tile of X (one reduction block of 128 rows).  One thread
// brings the whole tile (32 KB of BF16) into shared memory with a single TMA load,
// row-major: 256 bytes per row, the layout the token-wise transpose reads.  No thread
// holds in-flight loads in registers, so five CTAs (five tiles' loads) share an SM.
//   ROWS: 1x128 groups along K (the tile's columns) -> q[M][K], s[K/128][M].  Half-warp
//         h of warp w holds rows 16p + 2w + h (p < 8), 8 values per lane: each lane's
//         partial amax for its 8 rows goes through a transposing reduction over the
//         16 lanes (recursive halving: exchange half of the rows' partials with the
//         lane 8, 4, 2 apart, then combine with the lane 1 apart), after which lanes
//         2p and 2p + 1 hold the amax of row 16p + rsub.  Each lane works out that one
//         group's scale (and reciprocal), and the quantizing loop fetches group p's
//         scalars by shuffle, so the per-group division and reciprocal run once per
//         lane for all 8 groups instead of once per group.
//   COLS: 1x128 groups along M (the tile's rows) -> qt[K][M], st[M/128][K]; thread t
//         takes column pair t%64 over rows 32*(t/64) .. +31 (conflict-free 4-byte
//         reads), the four row quarters meet in shared memory for the column absmax,
//         and a second sweep quantizes.
// With both, X is read once for the two layouts wgrad and fprop/dgrad need.
// E8: power-of-two scales in 512-byte blocks (see sf_block_off): s holds
// [M/128][K/128] blocks (row m of block (m/128, kb)), st holds [K/128][M/128] blocks
// (column k of X is row k % 128 of block (k/128, mb)).
constexpr int QD_THREADS = 256;
constexpr int QD_MIN_BLOCKS = 5;  // at most 48 registers

__device__ int g_quant_error;  // first error code of a bounded wait in the quantizers
constexpr int QERR_TILE_LOAD = 21;
constexpr uint64_t QT_WAIT_NS = 1000000000ull;
constexpr uint64_t QT_DRAIN_NS = 20000000ull;

// RAGGED: M is not a multiple of 128, so the last row tile is partial and the stores
// past M are skipped; whole tiles run the unguarded instantiation.
template <bool ROWS, bool COLS, bool E8, bool RAGGED>
__global__ void __launch_bounds__(QD_THREADS, QD_MIN_BLOCKS)
quant_tile_kernel(const __grid_constant__ CUtensorMap tmX, int64_t M, int64_t K,
                      uint2 *__restrict__ q, void *__restrict__ s_out, uint8_t *__restrict__ qt,
                      void *__restrict__ st_out)
{
    __shared__ __align__(128) uint32_t tile[128 * 64];
    __shared__ uint32_t red[4][64];
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    const int t = threadIdx.x;
    const int64_t kb = blockIdx.x, mb = blockIdx.y;
    const int rsub = t >> 4, sub = t & 15;

    pdl_wait();               // X (and the output buffers) are free of the previous kernel
    pdl_launch_dependents();
    if (t == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbarrier_init();
        mbar_arrive_expect_tx(&bar, 128 * 128 * 2);
        tma_load_2d(tile, &tmX, &bar, int32_t(kb * 128), int32_t(mb * 128));
    }
    __syncthreads();
    const bool loaded =
        mbar_wait_bounded(&bar, 0u, &abort_flag, &g_quant_error, QERR_TILE_LOAD, QT_WAIT_NS);
    // Block-uniform decision: every thread leaves, or none does, so the barriers and
    // full-warp shuffles below never run with exited threads.
    if (__syncthreads_or(!loaded)) {
        if (t == 0) {  // keep the CTA (and its shared memory) alive while the copy may land
            const uint64_t t0 = global_timer_ns();
            while (global_timer_ns() - t0 < QT_DRAIN_NS) {
            }
        }
        return;
    }
    const uint4 *tile4 = reinterpret_cast<const uint4 *>(tile);  // [128 rows][16 uint4]

    if (ROWS) {
        uint32_t mx[8];
#pragma unroll
        for (int p = 0; p < 8; ++p) {
            const uint4 v = tile4[(p * 16 + rsub) * 16 + sub];
            mx[p] = __vmaxu2(absmax2(v.x, v.y), absmax2(v.z, v.w));
        }
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
        float g0 = 0.0f, g1 = 0.0f;
        if constexpr (E8) {
            const int e = e8m0_exponent(amax);
            g0 = amax != 0.0f ? pow2_neg(e) : 0.0f;
            if ((sub & 1) == 0 && (!RAGGED || m_own < M))
                *reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(s_out) +
                                              ((m_own >> 7) * (K / 128) + kb) * 512 +
                                              sf_block_off(int(m_own & 127))) = rep4_code(e, amax);
        } else {
            g0 = scale_of_amax(amax);
            const GroupDiv d(g0);
            g1 = d.fast ? d.r : -1.0f;
            if ((sub & 1) == 0 && (!RAGGED || m_own < M))
                static_cast<float *>(s_out)[kb * M + m_own] = g0;
        }
#pragma unroll
        for (int p = 0; p < 8; ++p) {
            const int64_t m = mb * 128 + p * 16 + rsub;
            const float gp = __shfl_sync(0xffffffffu, g0, 2 * p, 16);
            const uint4 v = tile4[(p * 16 + rsub) * 16 + sub];
            uint2 codes = make_uint2(0u, 0u);
            if constexpr (E8) {
                if (gp != 0.0f)
                    codes = quant8_pow2(v, gp);
            } else {
                const float rp = __shfl_sync(0xffffffffu, g1, 2 * p, 16);
                if (gp != 0.0f)
                    codes = rp > 0.0f ? quant8_fast(v, rp, gp) : quant8_ieee(v, gp);
            }
            if (!RAGGED || m < M)  // rows past M (a partial last tile) read as zeros: not stored
                q[(m * K + kb * 128) / 8 + sub] = codes;
        }
    }
    if (COLS) {
        // Token groups: thread t takes column pair t % 64 over rows 32 (t / 64) .. +31;
        // a first sweep for the column amax, a second to quantize.
        const int cp = t & 63, rq = t >> 6;
        const uint32_t *col = tile + (rq * 32) * 64 + cp;
        uint32_t m2 = 0;
#pragma unroll
        for (int i = 0; i < 32; i += 2)
            m2 = __vmaxu2(m2, absmax2(col[i * 64], col[(i + 1) * 64]));
        red[rq][cp] = m2;
        __syncthreads();
        m2 = __vmaxu2(__vmaxu2(red[0][cp], red[1][cp]), __vmaxu2(red[2][cp], red[3][cp]));
        const float amax_lo = __uint_as_float((m2 & 0xFFFFu) << 16);
        const float amax_hi = __uint_as_float(m2 & 0xFFFF0000u);
        const float s_lo = E8 ? 0.0f : scale_of_amax(amax_lo);
        const float s_hi = E8 ? 0.0f : scale_of_amax(amax_hi);
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
                const uint32_t w0 = col[i * 64], w1 = col[(i + 1) * 64];
                const float2 a = __fmul2_rn(make_float2(bf16lo(w0), bf16hi(w0)), mul2);
                const float2 b = __fmul2_rn(make_float2(bf16lo(w1), bf16hi(w1)), mul2);
                clo[i / 4] |= cvt_e4m3x2(a.x, b.x) << (16 * ((i / 2) & 1));
                chi[i / 4] |= cvt_e4m3x2(a.y, b.y) << (16 * ((i / 2) & 1));
            }
        } else if (dlo.fast && dhi.fast) {
            const float2 r2 = make_float2(dlo.r, dhi.r), nr2 = make_float2(-dlo.r, -dhi.r);
            const float2 s2 = make_float2(s_lo, s_hi);
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
                const uint32_t w0 = col[i * 64], w1 = col[(i + 1) * 64];
                const float2 a = div2_fast(make_float2(bf16lo(w0), bf16hi(w0)), r2, nr2, s2);
                const float2 b = div2_fast(make_float2(bf16lo(w1), bf16hi(w1)), r2, nr2, s2);
                clo[i / 4] |= cvt_e4m3x2(a.x, b.x) << (16 * ((i / 2) & 1));
                chi[i / 4] |= cvt_e4m3x2(a.y, b.y) << (16 * ((i / 2) & 1));
            }
        } else {
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
                const uint32_t w0 = col[i * 64], w1 = col[(i + 1) * 64];
                clo[i / 4] |= cvt_e4m3x2(__fdiv_rn(bf16lo(w0), s_lo), __fdiv_rn(bf16lo(w1), s_lo))
                              << (16 * ((i / 2) & 1));
                chi[i / 4] |= cvt_e4m3x2(__fdiv_rn(bf16hi(w0), s_hi), __fdiv_rn(bf16hi(w1), s_hi))
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
        const int64_t c = kb * 128 + 2 * cp;
        const int64_t m0 = mb * 128 + rq * 32;
        uint4 *dlo_p = reinterpret_cast<uint4 *>(qt + c * M + m0);
        uint4 *dhi_p = reinterpret_cast<uint4 *>(qt + (c + 1) * M + m0);
        // A partial last token group (M a multiple of 16): rows past M read as zeros
        // (no effect on the amax) and their 16-byte pieces of qt are not stored.
        if (!RAGGED || m0 < M) {
            dlo_p[0] = make_uint4(clo[0], clo[1], clo[2], clo[3]);
            dhi_p[0] = make_uint4(chi[0], chi[1], chi[2], chi[3]);
        }
        if (!RAGGED || m0 + 16 < M) {
            dlo_p[1] = make_uint4(clo[4], clo[5], clo[6], clo[7]);
            dhi_p[1] = make_uint4(chi[4], chi[5], chi[6], chi[7]);
        }
        if (rq == 0) {
            if (E8) {
                uint8_t *blk = static_cast<uint8_t *>(st_out) + ((c >> 7) * (M / 128) + mb) * 512;
                *reinterpret_cast<uint32_t *>(blk + sf_block_off(int(c & 127))) = rep4_code(e_lo, amax_lo);
                *reinterpret_cast<uint32_t *>(blk + sf_block_off(int((c + 1) & 127))) = rep4_code(e_hi, amax_hi);
            } else
                *reinterpret_cast<float2 *>(static_cast<float *>(st_out) + mb * K + c) =
                    make_float2(s_lo, s_hi);
        }
    }
}

typedef CUresult (*QEncodeFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                              const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                              const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                              CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// BF16 [M][K] map with 128 x 128 boxes, no swizzle (rows of 256 bytes).
static bool tile_map_bf16(CUtensorMap *map, const void *x, int64_t M, int64_t K)
{
    static QEncodeFn enc = [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult r;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                             &r) != cudaSuccess ||
            r != cudaDriverEntryPointSuccess)
            p = nullptr;
        return reinterpret_cast<QEncodeFn>(p);
    }();
    if (!enc)
        return false;
    cuuint64_t gdim[2] = {cuuint64_t(K), cuuint64_t(M)};
    cuuint64_t gstride[1] = {cuuint64_t(K) * 2};
    cuuint32_t box[2] = {128, 128};
    cuuint32_t estride[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(x), gdim, gstride, box,
               estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool ROWS, bool COLS, bool E8>
static cudaError_t run_tile(const void *x, int64_t M, int64_t K, void *q, void *s, uint8_t *qt,
                                void *st, cudaStream_t stream)
{
    CUtensorMap map;
    if (!tile_map_bf16(&map, x, M, K))
        return cudaErrorInvalidValue;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute at[1];
    set_pdl(at[0]);
    cfg.gridDim = dim3(unsigned(K / 128), unsigned((M + 127) / 128));  // last tile may be partial
    cfg.blockDim = dim3(QD_THREADS);
    cfg.stream = stream;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg,
                                       (M % 128) ? quant_tile_kernel<ROWS, COLS, E8, true>
                                                 : quant_tile_kernel<ROWS, COLS, E8, false>,
                                       map, M, K,
                                       reinterpret_cast<uint2 *>(q), s, qt, st);
    return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t read_and_clear_quant_error(int *value)
{
    cudaError_t e = cudaMemcpyFromSymbol(value, g_quant_error, sizeof(int));
    if (e != cudaSuccess)
        return e;
    if (*value) {
        const int zero = 0;
        e = cudaMemcpyToSymbol(g_quant_error, &zero, sizeof(int));
    }
    return e;
}

template <bool E8>
static cudaError_t run_weight(const void *w, int64_t N, int64_t K, void *q, void *s, uint8_t *qt,
                              cudaStream_t stream)
{
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute at[1];
    set_pdl(at[0]);
    cfg.gridDim = dim3(unsigned(K / 128), unsigned(N / 128));
    cfg.blockDim = dim3(QW_THREADS);
    cfg.stream = stream;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, quant_weight_kernel<E8>, static_cast<const uint4 *>(w),
                                       N, K, reinterpret_cast<uint2 *>(q), s, qt);
    return e != cudaSuccess ? e : cudaGetLastError();
}

// ------------------------------------------------------------------ launchers

cudaError_t launch_quant_act(const void *x, int64_t M, int64_t K, uint8_t *q, float *s,
                             cudaStream_t stream, int /*num_sms*/)
{
    return run_tile<true, false, false>(x, M, K, q, s, nullptr, nullptr, stream);
}

cudaError_t launch_quant_dual(const void *x, int64_t M, int64_t K, uint8_t *q, float *s,
                              uint8_t *qt, float *st, cudaStream_t stream)
{
    return run_tile<true, true, false>(x, M, K, q, s, qt, st, stream);
}

cudaError_t launch_quant_act_t(const void *x, int64_t M, int64_t K, uint8_t *qt, float *st,
                               cudaStream_t stream)
{
    return run_tile<false, true, false>(x, M, K, nullptr, nullptr, qt, st, stream);
}

cudaError_t launch_quant_weight(const void *w, int64_t N, int64_t K, uint8_t *q, float *s,
                                uint8_t *qt, cudaStream_t stream)
{
    return run_weight<false>(w, N, K, q, s, qt, stream);
}

// Power-of-two (E8M0) scale quantizers: the same code layouts, scales as 512-byte
// tensor-core scale blocks.
cudaError_t launch_quant_e8m0(int which, const void *x, int64_t M, int64_t K, uint8_t *q,
                              uint8_t *s, uint8_t *qt, uint8_t *st, cudaStream_t stream)
{
    switch (which) {
    case 0:  // rows: q[M][K], s[K/128][M]
        return run_tile<true, false, true>(x, M, K, q, s, nullptr, nullptr, stream);
    case 1:  // token groups: qt[K][M], st[M/128][K]
        return run_tile<false, true, true>(x, M, K, nullptr, nullptr, qt, st, stream);
    case 2:  // both
        return run_tile<true, true, true>(x, M, K, q, s, qt, st, stream);
    default: {  // weight blocks: q[N=M][K], s[M/128][K/128], optional qt[K][M]
        return run_weight<true>(x, M, K, q, s, qt, stream);
    }
    }
}

} // namespace fp8bw
