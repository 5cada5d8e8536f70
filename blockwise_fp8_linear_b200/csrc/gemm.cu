// gemm.cu -- blockwise-scaled FP8 GEMM on the 5th-generation tensor cores (sm_100a).
//
// D[M][N] (BF16) = sum over 128-long reduction blocks kb of
//     (a-scale x b-scale of kb) * (sum_{k in kb} qa[m][k] * qb[n][k]),
// the fprop / dgrad / wgrad GEMMs of the FP8 linear layer (Puro-2B part 3/7,
// section 3.2: all three GEMMs use the FP8 path, with FP32 accumulation and a BF16
// result handed back to the model).
//
// Design (one persistent CTA per SM, warp-specialised):
//   warp 0      TMA producer: 128x128 A tile + BNx128 B tile per stage, 128-byte
//               swizzle, STAGES-deep ring of shared-memory stages.
//   warp 1      MMA issuer: per reduction block, 4 x tcgen05.mma kind::f8f6f4
//               (K = 32 each) into one of two TMEM partial buffers (fresh
//               accumulation per block), then commits to the stage's "empty" barrier
//               and to the buffer's "full" barrier.
//   warps 2..3  idle (they complete the first warpgroup, which gives registers away)
//   warps 4..11 promotion + epilogue: each thread owns one TMEM lane (a row of the
//               tile) and COLS columns.  Per block it loads the FP32 partial from TMEM,
//               releases the buffer, and adds partial * scale into an FP32 running sum
//               held in registers (packed f32x2 FMA).  After the last block it rounds
//               the sum to BF16 and stores it.
// Double-buffered TMEM partials let the tensor cores run block kb+1 while the
// epilogue promotes block kb.  Every wait is bounded (about one second); a wait that
// runs out records an error code and the whole block unwinds.
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "ptx.cuh"
#include "quant.cuh"

namespace fp8bw {

__device__ int g_device_error;  // first error code seen by a bounded wait (0 = none)

constexpr int BM = 128;
constexpr int BK = 128;
constexpr uint64_t WAIT_LIMIT_NS = 1000000000ull;
constexpr uint64_t DRAIN_LIMIT_NS = 100000000ull;

enum : int { ERR_PRODUCER = 1, ERR_MMA_FULL = 2, ERR_MMA_TEMPTY = 3, ERR_EPI = 4, ERR_DRAIN = 5 };

template <int BN_, int MODE_, int STAGES_>
struct GemmCfg {
    static constexpr int BN = BN_;
    static constexpr int MODE = MODE_;  // 0 fprop, 1 dgrad (B is MN-major), 2 wgrad
    static constexpr int STAGES = STAGES_;
    static constexpr int EPI_WARPS = 8;
    static constexpr int COLS = 4 * BN / EPI_WARPS;  // columns per epilogue thread
    static constexpr int THREADS = 128 + 32 * EPI_WARPS;  // 3 warpgroups
    static constexpr int EPI_WARP0 = 4;
    // setmaxnreg split: the first warpgroup drops to REGS_LOW, the two epilogue
    // warpgroups rise to REGS_HIGH.  The host checks that the launch allocation
    // (ptxas register count x THREADS) covers REGS_NEEDED before launching.
    static constexpr int REGS_LOW = 72;
    static constexpr int REGS_HIGH = 216;
    static constexpr int REGS_NEEDED = 128 * REGS_LOW + 32 * EPI_WARPS * REGS_HIGH;
    static constexpr int A_BYTES = BM * BK;
    static constexpr int B_BYTES = BN * BK;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int TMEM_COLS = 2 * BN;
    static constexpr int SBV_BYTES = (MODE == 2) ? EPI_WARPS * COLS * 4 : 0;
    static constexpr int BAR_OFF = STAGES * STAGE_BYTES + SBV_BYTES;
    static constexpr int SMEM = 1024 + BAR_OFF + 256;
    static_assert(COLS % 32 == 0, "columns per thread must be whole TMEM load chunks");
    static_assert(BN % 128 == 0 && BN <= 256, "BN must be 128 or 256");
    static_assert(SMEM <= 227 * 1024, "shared memory budget");
};

// Tile t -> (tm, tn): column-major over groups of GROUP_M row-tiles, so the CTAs
// running at one time share A rows and B columns in L2.
constexpr int GROUP_M = 16;

__device__ __forceinline__ void tile_coords(int t, int tiles_m, int tiles_n, int &tm, int &tn)
{
    const int per_group = GROUP_M * tiles_n;
    const int g = t / per_group;
    const int first = g * GROUP_M;
    const int gsize = min(GROUP_M, tiles_m - first);
    const int r = t - g * per_group;
    tm = first + r % gsize;
    tn = r / gsize;
}

template <class Cfg>
__global__ void __launch_bounds__(Cfg::THREADS, 1)
fp8_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const float *__restrict__ sa, const float *__restrict__ sb,
                __nv_bfloat16 *__restrict__ D, int M, int N, int K)
{
    constexpr int BN = Cfg::BN, MODE = Cfg::MODE, STAGES = Cfg::STAGES;
    constexpr int COLS = Cfg::COLS, EPI_WARPS = Cfg::EPI_WARPS;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float *sbv = reinterpret_cast<float *>(smem + STAGES * Cfg::STAGE_BYTES);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::BAR_OFF);
    uint64_t *full = bars;                 // [STAGES] TMA -> MMA
    uint64_t *empty = bars + STAGES;       // [STAGES] MMA -> TMA
    uint64_t *tfull = bars + 2 * STAGES;   // [2] MMA -> epilogue
    uint64_t *tempty = tfull + 2;          // [2] epilogue -> MMA
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tempty + 2);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tiles_m = M / BM, tiles_n = N / BN;
    const int num_tiles = tiles_m * tiles_n;
    const int KB = K / BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], EPI_WARPS);
        }
        *abort_flag = 0;
        fence_mbarrier_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    // Producer / MMA state kept for the drain after an abort.
    uint32_t armed_mask = 0, armed_parity = 0;  // producer: stages with a load in flight
    int last_buf = -1;
    uint32_t last_tparity = 0;                  // MMA: last commit to tfull

    if (warp < Cfg::EPI_WARP0) {
      regs_dec<Cfg::REGS_LOW>();
      if (warp == 0) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            for (int t = blockIdx.x; t < num_tiles && !*abort_flag; t += gridDim.x) {
                int tm, tn;
                tile_coords(t, tiles_m, tiles_n, tm, tn);
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag, &g_device_error,
                                           ERR_PRODUCER, WAIT_LIMIT_NS))
                        goto producer_done;
                    uint8_t *sA = smem + stage * Cfg::STAGE_BYTES;
                    uint8_t *sB = sA + Cfg::A_BYTES;
                    mbar_arrive_expect_tx(&full[stage], Cfg::STAGE_BYTES);
                    armed_mask |= 1u << stage;
                    armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
                    tma_load_2d(sA, &tmA, &full[stage], kb * BK, tm * BM);
                    if (MODE == 1) {
                        // B = W[K][N] with N contiguous: BN/128 boxes of 128 (N) x 128 (K).
#pragma unroll
                        for (int j = 0; j < BN / 128; ++j)
                            tma_load_2d(sB + j * 128 * BK, &tmB, &full[stage], tn * BN + j * 128,
                                        kb * BK);
                    } else {
                        tma_load_2d(sB, &tmB, &full[stage], kb * BK, tn * BN);
                    }
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
        producer_done:;
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = make_idesc_e4m3(BM, BN, MODE == 1 ? 1 : 0);
            int stage = 0, buf = 0;
            uint32_t phase = 0, tphase = 0;
            for (int t = blockIdx.x; t < num_tiles && !*abort_flag; t += gridDim.x) {
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait_bounded(&full[stage], phase, abort_flag, &g_device_error,
                                           ERR_MMA_FULL, WAIT_LIMIT_NS))
                        goto mma_done;
                    if (!mbar_wait_bounded(&tempty[buf], tphase ^ 1u, abort_flag, &g_device_error,
                                           ERR_MMA_TEMPTY, WAIT_LIMIT_NS))
                        goto mma_done;
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(smem + stage * Cfg::STAGE_BYTES);
                    const uint32_t b_addr = a_addr + Cfg::A_BYTES;
                    const uint32_t d_tmem = tmem_base + uint32_t(buf * BN);
#pragma unroll
                    for (int k = 0; k < BK / 32; ++k) {
                        // K-major, 128B swizzle: rows 128 B apart, 8-row atoms 1024 B apart;
                        // a K step of 32 bytes moves the start address by 32 B.
                        const uint64_t adesc = make_smem_desc_sw128(a_addr + k * 32, 16, 1024);
                        uint64_t bdesc;
                        if (MODE == 1) {
                            // MN-major, 128B swizzle: 128 N-bytes per row, one row per k;
                            // atoms of 8 k-rows 1024 B apart (SBO), 128-wide N atoms
                            // 16 KB apart (LBO); a K step of 32 rows moves 4 KB.
                            bdesc = make_smem_desc_sw128(b_addr + k * 32 * 128, 128 * BK, 1024);
                        } else {
                            bdesc = make_smem_desc_sw128(b_addr + k * 32, 16, 1024);
                        }
                        mma_f8f6f4(d_tmem, adesc, bdesc, idesc, k > 0 ? 1u : 0u);
                    }
                    mma_commit(&empty[stage]);
                    mma_commit(&tfull[buf]);
                    last_buf = buf;
                    last_tparity = tphase;
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                    if (++buf == 2) {
                        buf = 0;
                        tphase ^= 1u;
                    }
                }
            }
        mma_done:;
        }
      }
    } else {
        regs_inc<Cfg::REGS_HIGH>();
        // ---------------------------------------------------- promotion + epilogue
        const int ew = warp - Cfg::EPI_WARP0;
        const int quarter = warp & 3;           // TMEM lanes this warp may access
        const int col0 = (ew >> 2) * COLS;      // columns of the tile this thread owns
        const int row_in_tile = quarter * 32 + lane;
        float *my_sbv = sbv + ew * COLS;        // wgrad: this warp's column scales

        float2 acc[COLS / 2];
#pragma unroll
        for (int i = 0; i < COLS / 2; ++i)
            acc[i] = make_float2(0.f, 0.f);

        // Scales of iteration j = (tile index i, block kb), fetched two iterations
        // ahead.  For fprop/dgrad the thread needs one a-scale (its row) and one
        // b-scale (its 128-column block); for wgrad one a-scale and COLS b-scales,
        // which lanes load cooperatively (COLS/32 per lane) into shared memory.
        constexpr int VB = (MODE == 2) ? COLS / 32 : 1;
        const int total_iters = ((num_tiles - int(blockIdx.x) + int(gridDim.x) - 1) /
                                 int(gridDim.x)) * KB;
        auto fetch = [&](int j, float &a_out, float (&b_out)[VB]) {
            if (j >= total_iters)
                return;
            const int i = j / KB, kb = j - i * KB;
            int tm, tn;
            tile_coords(int(blockIdx.x) + i * int(gridDim.x), tiles_m, tiles_n, tm, tn);
            a_out = __ldg(sa + size_t(kb) * M + tm * BM + row_in_tile);
            const int ncol = tn * BN + col0;
            if (MODE == 0) {
                b_out[0] = __ldg(sb + size_t(ncol / 128) * KB + kb);
            } else if (MODE == 1) {
                b_out[0] = __ldg(sb + size_t(kb) * (N / 128) + ncol / 128);
            } else {
                const float *p = sb + size_t(kb) * N + ncol + lane * VB;
#pragma unroll
                for (int v = 0; v < VB; ++v)
                    b_out[v] = __ldg(p + v);
            }
        };
        float a0 = 0.f, a1 = 0.f, a2 = 0.f;
        float b0[VB], b1[VB], b2[VB];
#pragma unroll
        for (int v = 0; v < VB; ++v)
            b0[v] = b1[v] = b2[v] = 0.f;
        fetch(0, a0, b0);
        fetch(1, a1, b1);

        int buf = 0;
        uint32_t tphase = 0;
        for (int j = 0; j < total_iters; ++j) {
            fetch(j + 2, a2, b2);
            const int i = j / KB, kb = j - i * KB;
            if (MODE == 2) {
#pragma unroll
                for (int v = 0; v < VB; ++v)
                    my_sbv[lane * VB + v] = b0[v];
                __syncwarp();
            }
            const bool ready = mbar_wait_bounded(&tfull[buf], tphase, abort_flag,
                                                 &g_device_error, ERR_EPI, WAIT_LIMIT_NS);
            if (!__all_sync(0xffffffffu, ready))  // leave together: tcgen05.ld is warp-wide
                break;
            tc_fence_after();
            const uint32_t taddr =
                tmem_base + (uint32_t(quarter * 32) << 16) + uint32_t(buf * BN + col0);
            const float sc = a0 * b0[0];
            const float2 sc2 = make_float2(sc, sc);
            const float2 sa2 = make_float2(a0, a0);
            constexpr int CHUNKS = COLS / 32;
            constexpr int GROUP = 1;  // TMEM loads in flight per wait
            static_assert(CHUNKS % GROUP == 0, "chunk grouping");
#pragma unroll
            for (int cg = 0; cg < CHUNKS; cg += GROUP) {
                uint32_t v[GROUP][32];
#pragma unroll
                for (int g = 0; g < GROUP; ++g)
                    tmem_ld_32x32b_x32(taddr + uint32_t((cg + g) * 32), v[g]);
                tmem_wait_ld();
                if (cg + GROUP == CHUNKS) {
                    // Partial fully in registers: hand the TMEM buffer back to the MMA.
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive(&tempty[buf]);
                }
#pragma unroll
                for (int g = 0; g < GROUP; ++g) {
                    const int c = cg + g;
#pragma unroll
                    for (int jj = 0; jj < 16; ++jj) {
                        const float2 p = make_float2(__uint_as_float(v[g][2 * jj]),
                                                     __uint_as_float(v[g][2 * jj + 1]));
                        if (MODE == 2) {
                            const float2 bs = *reinterpret_cast<const float2 *>(
                                my_sbv + c * 32 + 2 * jj);
                            acc[c * 16 + jj] =
                                __ffma2_rn(__fmul2_rn(p, bs), sa2, acc[c * 16 + jj]);
                        } else {
                            acc[c * 16 + jj] = __ffma2_rn(p, sc2, acc[c * 16 + jj]);
                        }
                    }
                }
            }
            if (MODE == 2)
                __syncwarp();  // all lanes done reading my_sbv before it is rewritten
            if (kb == KB - 1) {
                int tm, tn;
                tile_coords(int(blockIdx.x) + i * int(gridDim.x), tiles_m, tiles_n, tm, tn);
                __nv_bfloat16 *dst =
                    D + size_t(tm * BM + row_in_tile) * size_t(N) + size_t(tn * BN + col0);
#pragma unroll
                for (int c = 0; c < COLS / 8; ++c) {
                    uint4 o;
                    __nv_bfloat162 h0 = __float22bfloat162_rn(acc[4 * c + 0]);
                    __nv_bfloat162 h1 = __float22bfloat162_rn(acc[4 * c + 1]);
                    __nv_bfloat162 h2 = __float22bfloat162_rn(acc[4 * c + 2]);
                    __nv_bfloat162 h3 = __float22bfloat162_rn(acc[4 * c + 3]);
                    o.x = *reinterpret_cast<uint32_t *>(&h0);
                    o.y = *reinterpret_cast<uint32_t *>(&h1);
                    o.z = *reinterpret_cast<uint32_t *>(&h2);
                    o.w = *reinterpret_cast<uint32_t *>(&h3);
                    *reinterpret_cast<uint4 *>(dst + c * 8) = o;
                }
#pragma unroll
                for (int q = 0; q < COLS / 2; ++q)
                    acc[q] = make_float2(0.f, 0.f);
            }
            a0 = a1;
            a1 = a2;
#pragma unroll
            for (int v = 0; v < VB; ++v) {
                b0[v] = b1[v];
                b1[v] = b2[v];
            }
            if (++buf == 2) {
                buf = 0;
                tphase ^= 1u;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (*abort_flag) {
        // Unwind: let every load and MMA still in flight land before the block's
        // shared memory and tensor memory are released.
        if (warp == 0 && lane == 0) {
            for (int s = 0; s < STAGES; ++s)
                if (armed_mask & (1u << s))
                    mbar_wait_bounded(&full[s], (armed_parity >> s) & 1u, abort_flag,
                                      &g_device_error, ERR_DRAIN, DRAIN_LIMIT_NS);
        }
        if (warp == 1 && lane == 0 && last_buf >= 0) {
            // The flag is already set, so poll directly with a time limit.
            uint64_t t0 = global_timer_ns();
            while (!mbar_try_wait(&tfull[last_buf], last_tparity) &&
                   global_timer_ns() - t0 < DRAIN_LIMIT_NS) {
            }
        }
        __syncthreads();
    }
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
    }
}

// ------------------------------------------------------------------- host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode_fn()
{
    static EncodeTiledFn fn = [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                             &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            p = nullptr;
        return reinterpret_cast<EncodeTiledFn>(p);
    }();
    return fn;
}

// 2-D uint8 tensor map over a row-major [rows][cols] array, box {box_cols, box_rows},
// 128-byte swizzle.
static bool make_map_u8(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols,
                        uint32_t box_rows, uint32_t box_cols)
{
    EncodeTiledFn enc = get_encode_fn();
    if (!enc)
        return false;
    cuuint64_t gdim[2] = {cols, rows};
    cuuint64_t gstride[1] = {cols};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estride[2] = {1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), gdim, gstride,
                     box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <class Cfg>
static cudaError_t run(const uint8_t *a, const float *sa, const uint8_t *b, const float *sb,
                       void *d, int64_t M, int64_t N, int64_t K, cudaStream_t stream, int num_sms)
{
    auto kern = fp8_gemm_kernel<Cfg>;
    cudaFuncAttributes attr;
    cudaError_t e = cudaFuncGetAttributes(&attr, kern);
    if (e != cudaSuccess)
        return e;
    // setmaxnreg.inc waits until enough registers are free; refuse to launch a
    // split the launch allocation cannot cover (it would never make progress).
    if (attr.numRegs * Cfg::THREADS < Cfg::REGS_NEEDED)
        return cudaErrorInvalidConfiguration;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM);
    if (e != cudaSuccess)
        return e;
    CUtensorMap ta, tb;
    if (!make_map_u8(&ta, a, uint64_t(M), uint64_t(K), BM, BK))
        return cudaErrorInvalidValue;
    bool ok;
    if (Cfg::MODE == 1)
        ok = make_map_u8(&tb, b, uint64_t(K), uint64_t(N), BK, 128);  // W[K][N], N contiguous
    else
        ok = make_map_u8(&tb, b, uint64_t(N), uint64_t(K), Cfg::BN, BK);
    if (!ok)
        return cudaErrorInvalidValue;
    const int64_t tiles = (M / BM) * (N / Cfg::BN);
    const int grid = int(tiles < num_sms ? tiles : num_sms);
    fp8_gemm_kernel<Cfg><<<grid, Cfg::THREADS, Cfg::SMEM, stream>>>(
        ta, tb, sa, sb, static_cast<__nv_bfloat16 *>(d), int(M), int(N), int(K));
    return cudaGetLastError();
}

cudaError_t launch_gemm(int mode, const uint8_t *a, const float *sa, const uint8_t *b,
                        const float *sb, void *d, int64_t M, int64_t N, int64_t K,
                        cudaStream_t stream, int num_sms)
{
    const bool wide = (N % 256) == 0;
    switch (mode) {
    case 0:
        return wide ? run<GemmCfg<256, 0, 4>>(a, sa, b, sb, d, M, N, K, stream, num_sms)
                    : run<GemmCfg<128, 0, 6>>(a, sa, b, sb, d, M, N, K, stream, num_sms);
    case 1:
        return wide ? run<GemmCfg<256, 1, 4>>(a, sa, b, sb, d, M, N, K, stream, num_sms)
                    : run<GemmCfg<128, 1, 6>>(a, sa, b, sb, d, M, N, K, stream, num_sms);
    default:
        return wide ? run<GemmCfg<256, 2, 4>>(a, sa, b, sb, d, M, N, K, stream, num_sms)
                    : run<GemmCfg<128, 2, 6>>(a, sa, b, sb, d, M, N, K, stream, num_sms);
    }
}

cudaError_t read_and_clear_device_error(cudaStream_t stream, int *value)
{
    cudaError_t e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess)
        return e;
    e = cudaMemcpyFromSymbol(value, g_device_error, sizeof(int));
    if (e != cudaSuccess)
        return e;
    if (*value) {
        const int zero = 0;
        e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int));
    }
    return e;
}

} // namespace fp8bw
