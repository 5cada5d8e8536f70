// gemm_mx.cu -- the blockwise FP8 GEMM with power-of-two (E8M0) scales, promoted by
// the tensor cores themselves (sm_100a, tcgen05.mma kind::mxf8f6f4.block_scale).
//
// Puro-2B part 3/7, section 3.2: on its GPUs the recipe's 128-blocks run through the
// MXFP8 path, where every block scale is a power of two.  With such scales the
// hardware applies them inside the MMA: each K = 32 step multiplies its products by
// 2^(ea + eb) read from tensor memory, so the whole reduction accumulates in one
// TMEM accumulator and no per-block promotion runs on the CUDA cores.  The 1x128 /
// 128x128 scales of the recipe are simply repeated over the four 32-wide K steps of
// each 128-block.
//
//   D[M][N] (BF16) = sum over k of (qa[m][k] 2^ea(m, k/128)) (qb[n][k] 2^eb(n, k/128))
//
// Design (persistent, warp-specialised, one CTA or CTA pair per tile):
//   warp 0      TMA producer: per 128-deep reduction block, the A and B tiles and
//               their scale blocks into one pipeline stage.  The E8M0 quantizers
//               store scales in the layout the tensor cores read them in (512-byte
//               blocks of 128 rows: row r's code at bytes 16 (r % 32) + 4 (r / 32),
//               repeated four times for the four 32-wide K steps), so scale factors
//               travel by TMA with the operands and need no rewriting on chip.
//   warp 1      MMA issuer (even CTA): per block, four block-scaled MMAs into the
//               tile's accumulator, reading the stage's scale factors from tensor memory.
//   warp 2      scale copier (even CTA): per block, tcgen05.cp of the stage's scale
//               blocks into that stage's tensor-memory region, so the MMA issuer's
//               thread issues nothing but MMAs and commits.
//   warps 4-11  epilogue: after the tile's last block, load the accumulator from TMEM,
//               release it to the MMA issuer, round to BF16 and store through swizzled
//               shared memory with TMA.
// Tensor memory: the accumulator (BN columns), then one 16-column region per pipeline
// stage holding 4 columns of A scale factors and 4 per 128 columns of B scale factors.
//
// Every wait is bounded (about one second); a wait that runs out records an error
// code and the CTA (pair) unwinds.
#include <cstdint>
#include <cstring>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "launch_cache.cuh"
#include "ptx.cuh"
#include "ptx_mx.cuh"
#include "quant.cuh"

namespace fp8bw {

namespace {

__device__ int g_mx_error;  // first error code seen by a bounded wait in this kernel

constexpr int MX_BM = 128;
constexpr int MX_BK = 128;
constexpr uint64_t MX_WAIT_NS = 1000000000ull;
constexpr uint64_t MX_DRAIN_NS = 20000000ull;

enum : int { MXE_PRODUCER = 11, MXE_MMA = 12, MXE_EPI = 14, MXE_TEMPTY = 15 };

template <int BN_, int MODE_, int CG_>
struct MxCfg {
    static constexpr int BN = BN_;
    static constexpr int MODE = MODE_;  // 0 fprop, 1 dgrad (B MN-major), 2 wgrad
    static constexpr int CG = CG_;
    static constexpr int TILE_M = MX_BM * CG;
    static constexpr int STAGES = 4;
    static constexpr int EPI_WARPS = 8;
    static constexpr int THREADS = 128 + 32 * EPI_WARPS;
    static constexpr int COLS = 4 * BN / EPI_WARPS;        // accumulator columns per thread
    static constexpr int B_ROWS = BN / CG;
    static constexpr int A_BYTES = MX_BM * MX_BK;
    static constexpr int B_BYTES = B_ROWS * MX_BK;
    static constexpr int B_BOX = 128;
    static constexpr int NSFB = BN / 128;                  // B scale blocks of 128 columns
    static constexpr int SF_BYTES = 512 * (1 + NSFB);      // A scale block, then the B ones
    static constexpr int LOAD_BYTES = A_BYTES + B_BYTES + SF_BYTES;  // per CTA and stage
    static constexpr int STAGE_BYTES = (LOAD_BYTES + 1023) / 1024 * 1024;
    static constexpr int OUT_WARP = 32 * COLS * 2;         // BF16 staging per epilogue warp
    static constexpr int OUT_OFF = STAGES * STAGE_BYTES;
    static constexpr int BAR_OFF = OUT_OFF + EPI_WARPS * OUT_WARP;
    static constexpr int SMEM = 1024 + BAR_OFF + 256;
    static constexpr int TMEM_COLS = 512;
    static constexpr int SF_COL = BN;                      // first scale-factor region
    static constexpr int SF_COLS = 16;                     // per stage: A (4), then B (4 each)
    static_assert(COLS % 64 == 0, "epilogue works in 64-column boxes");
    static_assert(B_ROWS % B_BOX == 0, "B rows must be whole boxes");
    static_assert(4 * (1 + NSFB) <= SF_COLS, "scale factors of one stage");
    static_assert(SF_COL + STAGES * SF_COLS <= TMEM_COLS, "tensor memory budget");
    static_assert(SMEM <= 227 * 1024, "shared memory budget");
};

constexpr int MX_GROUP_M = 16;

__device__ __forceinline__ void mx_tile_coords(int t, int tiles_m, int tiles_n, int &tm, int &tn)
{
    const int per_group = MX_GROUP_M * tiles_n;
    const int g = t / per_group;
    const int first = g * MX_GROUP_M;
    const int gsize = min(MX_GROUP_M, tiles_m - first);
    const int r = t - g * per_group;
    tm = first + r % gsize;
    tn = r / gsize;
}

// Scale blocks are indexed [rows/128][K/128] for A and for the B of fprop and wgrad;
// the B of dgrad is the weight, whose blocks are [K/128][N/128] in GEMM terms.
template <class Cfg>
__global__ void __launch_bounds__(Cfg::THREADS, 1)
fp8_gemm_mx_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmD, const __grid_constant__ CUtensorMap tmSA,
                   const __grid_constant__ CUtensorMap tmSB, int M, int N, int K)
{
    constexpr int BN = Cfg::BN, MODE = Cfg::MODE, STAGES = Cfg::STAGES, CG = Cfg::CG;
    constexpr int COLS = Cfg::COLS, EPI_WARPS = Cfg::EPI_WARPS;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sout = smem + Cfg::OUT_OFF;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::BAR_OFF);
    uint64_t *full = bars;                 // [STAGES] TMA -> MMA (even CTA)
    uint64_t *empty = full + STAGES;       // [STAGES] MMA -> TMA
    uint64_t *tfull = empty + STAGES;      // MMA -> epilogue
    uint64_t *tempty = tfull + 1;          // epilogue -> MMA (even CTA)
    uint64_t *sfr = tempty + 1;            // [STAGES] scale copier -> MMA (even CTA)
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sfr + STAGES);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rank = (CG == 2) ? int(cluster_ctarank()) : 0;
    const int unit = (CG == 2) ? int(cluster_id_x()) : int(blockIdx.x);
    const int units = (CG == 2) ? int(cluster_count_x()) : int(gridDim.x);
    const int tiles_m = M / Cfg::TILE_M, tiles_n = N / BN;
    const int num_tiles = tiles_m * tiles_n;
    const int KB = K / MX_BK;
    const int my_tiles = num_tiles > unit ? (num_tiles - unit + units - 1) / units : 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
            mbar_init(&sfr[s], 1);
        }
        mbar_init(tfull, 1);
        mbar_init(tempty, EPI_WARPS * CG);
        *abort_flag = 0;
        fence_mbarrier_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        tma_prefetch_desc(&tmSA);
        tma_prefetch_desc(&tmSB);
    }
    if (warp == 1) {
        tmem_alloc<CG>(tmem_slot, Cfg::TMEM_COLS);
        tmem_relinquish<CG>();
    }
    tc_fence_before();
    if (CG == 2)
        cluster_sync();
    else
        __syncthreads();
    tc_fence_after();
    pdl_wait();               // inputs written by the previous kernel are visible
    pdl_launch_dependents();  // the next kernel may start its launch and prologue
    const uint32_t tmem_base = *tmem_slot;
    const uint32_t full_lead = (CG == 2) ? mapa_shared(smem_u32(full), 0) : smem_u32(full);
    const uint32_t tempty_lead = (CG == 2) ? mapa_shared(smem_u32(tempty), 0) : smem_u32(tempty);

    if (warp < 4) {
        if (warp == 0 && lane == 0) {
            // ---------------------------------------------------------- producer
            int stage = 0;
            uint32_t phase = 0;
            for (int i = 0; i < my_tiles && !*abort_flag; ++i) {
                int tm, tn;
                mx_tile_coords(unit + i * units, tiles_m, tiles_n, tm, tn);
                const int arow = tm * Cfg::TILE_M + rank * MX_BM;
                const int bcol = tn * BN + rank * Cfg::B_ROWS;
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag, &g_mx_error,
                                           MXE_PRODUCER, MX_WAIT_NS))
                        goto role_done;
                    uint8_t *sA = smem + stage * Cfg::STAGE_BYTES;
                    uint8_t *sB = sA + Cfg::A_BYTES;
                    uint8_t *sS = sB + Cfg::B_BYTES;
                    // scale blocks: this CTA's 128 rows of A; all BN columns of B
                    const int sa_blk = (arow / MX_BM) * KB + kb;
                    int sb_blk[Cfg::NSFB];
#pragma unroll
                    for (int q = 0; q < Cfg::NSFB; ++q) {
                        const int nb = tn * Cfg::NSFB + q;
                        sb_blk[q] = (MODE == 1) ? kb * (N / 128) + nb : nb * KB + kb;
                    }
                    if (CG == 1) {
                        uint64_t *fb = &full[stage];
                        mbar_arrive_expect_tx(fb, Cfg::LOAD_BYTES);
                        tma_load_2d(sA, &tmA, fb, kb * MX_BK, arow);
                        if (MODE == 1) {
#pragma unroll
                            for (int j = 0; j < Cfg::B_ROWS / Cfg::B_BOX; ++j)
                                tma_load_2d(sB + j * Cfg::B_BOX * MX_BK, &tmB, fb, bcol + j * Cfg::B_BOX,
                                            kb * MX_BK);
                        } else {
                            tma_load_2d(sB, &tmB, fb, kb * MX_BK, bcol);
                        }
                        tma_load_2d(sS, &tmSA, fb, 0, sa_blk);
#pragma unroll
                        for (int q = 0; q < Cfg::NSFB; ++q)
                            tma_load_2d(sS + 512 * (1 + q), &tmSB, fb, 0, sb_blk[q]);
                    } else {
                        if (rank == 0)
                            mbar_arrive_expect_tx(&full[stage], 2 * Cfg::LOAD_BYTES);
                        const uint32_t fb = full_lead + uint32_t(stage) * 8u;
                        tma_load_2d_pair(sA, &tmA, fb, kb * MX_BK, arow);
                        if (MODE == 1) {
#pragma unroll
                            for (int j = 0; j < Cfg::B_ROWS / Cfg::B_BOX; ++j)
                                tma_load_2d_pair(sB + j * Cfg::B_BOX * MX_BK, &tmB, fb,
                                                 bcol + j * Cfg::B_BOX, kb * MX_BK);
                        } else {
                            tma_load_2d_pair(sB, &tmB, fb, kb * MX_BK, bcol);
                        }
                        tma_load_2d_pair(sS, &tmSA, fb, 0, sa_blk);
#pragma unroll
                        for (int q = 0; q < Cfg::NSFB; ++q)
                            tma_load_2d_pair(sS + 512 * (1 + q), &tmSB, fb, 0, sb_blk[q]);
                    }
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
        } else if (warp == 1 && lane == 0 && rank == 0) {
            // --------------------------------------------------------------- MMA
            int stage = 0;
            uint32_t phase = 0;
            const uint32_t d_tmem = tmem_base;
            for (int i = 0; i < my_tiles && !*abort_flag; ++i) {
                // the epilogue has drained the accumulator of the previous tile
                if (!mbar_wait_bounded(tempty, uint32_t(i & 1) ^ 1u, abort_flag, &g_mx_error,
                                       MXE_TEMPTY, MX_WAIT_NS))
                    goto role_done;
                for (int kb = 0; kb < KB; ++kb) {
                    // the stage's scale factors are in tensor memory (which implies its
                    // operands have landed); the full barrier is tested for the operands'
                    // own visibility and has completed by then
                    if (!mbar_spin_bounded(&sfr[stage], phase, abort_flag, &g_mx_error, MXE_MMA,
                                           MX_WAIT_NS) ||
                        !mbar_spin_bounded(&full[stage], phase, abort_flag, &g_mx_error, MXE_MMA,
                                           MX_WAIT_NS))
                        goto role_done;
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(smem + stage * Cfg::STAGE_BYTES);
                    const uint32_t b_addr = a_addr + Cfg::A_BYTES;
                    const uint32_t sfa_tmem = tmem_base + uint32_t(Cfg::SF_COL + stage * Cfg::SF_COLS);
                    const uint32_t sfb_tmem = sfa_tmem + 4;
#pragma unroll
                    for (int k = 0; k < MX_BK / 32; ++k) {
                        const uint64_t adesc = make_smem_desc_sw128(a_addr + k * 32, 16, 1024);
                        const uint64_t bdesc =
                            (MODE == 1) ? make_smem_desc_sw128(b_addr + k * 32 * 128, 128 * MX_BK, 1024)
                                        : make_smem_desc_sw128(b_addr + k * 32, 16, 1024);
                        constexpr int BMAJ = MODE == 1 ? 1 : 0;
                        const uint32_t idesc = make_idesc_mx_e4m3(Cfg::TILE_M, BN, BMAJ, k);
                        const uint32_t sel = uint32_t(k) << 30;  // byte k of each scale word
                        mma_mxf8f6f4<CG>(d_tmem, adesc, bdesc, idesc, sfa_tmem | sel, sfb_tmem | sel,
                                         (kb > 0 || k > 0) ? 1u : 0u);
                    }
                    if (CG == 1)
                        mma_commit(&empty[stage]);
                    else
                        mma_commit_pair(&empty[stage], 0x3);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (CG == 1)
                    mma_commit(tfull);
                else
                    mma_commit_pair(tfull, 0x3);
            }
        } else if (warp == 2 && lane == 0 && rank == 0) {
            // ---------------------------------------------------------- scale copier
            // Per stage: tcgen05.cp of its scale blocks into the stage's own tensor-memory
            // region, signalled to the MMA issuer by a commit.  A region is rewritten only
            // after the producer has seen the stage's MMAs complete (empty) and refilled it
            // (full), so the copy never overtakes the MMAs that read the previous contents.
            int stage = 0;
            uint32_t phase = 0;
            const int blocks = my_tiles * KB;
            for (int j = 0; j < blocks && !*abort_flag; ++j) {
                if (!mbar_spin_bounded(&full[stage], phase, abort_flag, &g_mx_error, MXE_MMA,
                                       MX_WAIT_NS))
                    goto role_done;
                tc_fence_after();
                const uint32_t sf_addr =
                    smem_u32(smem + stage * Cfg::STAGE_BYTES) + Cfg::A_BYTES + Cfg::B_BYTES;
                const uint32_t sfa_tmem = tmem_base + uint32_t(Cfg::SF_COL + stage * Cfg::SF_COLS);
                tmem_cp_32x128b_warpx4<CG>(sfa_tmem, make_smem_desc_rows16(sf_addr));
#pragma unroll
                for (int q = 0; q < Cfg::NSFB; ++q)
                    tmem_cp_32x128b_warpx4<CG>(sfa_tmem + 4 + 4 * q,
                                               make_smem_desc_rows16(sf_addr + 512 * (1 + q)));
                if (CG == 1)
                    mma_commit(&sfr[stage]);
                else
                    mma_commit_pair(&sfr[stage], 0x1);
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
    role_done:;
    } else {
        // ------------------------------------------------------------- epilogue
        const int ew = warp - 4;
        const int quarter = warp & 3;
        const int col0 = (ew >> 2) * COLS;
        uint8_t *stg = sout + ew * Cfg::OUT_WARP;
        for (int i = 0; i < my_tiles; ++i) {
            int tm, tn;
            mx_tile_coords(unit + i * units, tiles_m, tiles_n, tm, tn);
            const bool ready = mbar_spin_bounded(tfull, uint32_t(i & 1), abort_flag, &g_mx_error,
                                                 MXE_EPI, MX_WAIT_NS);
            if (!__all_sync(0xffffffffu, ready))
                break;
            tc_fence_after();
            const uint32_t taddr = tmem_base + (uint32_t(quarter * 32) << 16) + uint32_t(col0);
            uint32_t packed[COLS / 2];
#pragma unroll
            for (int c = 0; c < COLS / 64; ++c) {
                // one 64-column TMEM load per chunk (fewer, larger tcgen05.ld)
                uint32_t v[64];
                tmem_ld_32x32b_x64(taddr + uint32_t(64 * c), v);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(v[2 * e]),
                                                             __uint_as_float(v[2 * e + 1]));
                    packed[32 * c + e] = *reinterpret_cast<uint32_t *>(&h);
                }
            }
            // the accumulator is in registers: hand it back to the MMA issuer
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (CG == 1 || rank == 0)
                    mbar_arrive(tempty);
                else
                    mbar_arrive_cluster(tempty_lead);
            }
            // BF16 tile -> swizzled staging (64-column boxes of 32 rows x 128 B) -> TMA
            if (lane == 0)
                bulk_wait_read0();
            __syncwarp();
#pragma unroll
            for (int c = 0; c < COLS / 8; ++c) {
                const int box = c >> 3, chunk = c & 7;
                *reinterpret_cast<uint4 *>(stg + box * 4096 + lane * 128 + ((chunk ^ (lane & 7)) << 4)) =
                    make_uint4(packed[4 * c], packed[4 * c + 1], packed[4 * c + 2], packed[4 * c + 3]);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                const int r0 = tm * Cfg::TILE_M + rank * MX_BM + quarter * 32;
#pragma unroll
                for (int box = 0; box < COLS / 64; ++box)
                    tma_store_2d(&tmD, stg + box * 4096, tn * BN + col0 + box * 64, r0);
                bulk_commit();
            }
        }
        if (lane == 0)
            bulk_wait0();
    }

    tc_fence_before();
    __syncthreads();
    if (*abort_flag && threadIdx.x == 0) {
        const uint64_t t0 = global_timer_ns();
        while (global_timer_ns() - t0 < MX_DRAIN_NS) {
        }
    }
    if (CG == 2)
        cluster_sync();
    else
        __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc<CG>(tmem_base, Cfg::TMEM_COLS);
    }
}

// ----------------------------------------------------------------- host side

typedef CUresult (*EncodeFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                             const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                             const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                             CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeFn mx_encode_fn()
{
    static EncodeFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000,
                                             cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeFn>(p);
    }
    return fn;
}

static bool mx_map(CUtensorMap *map, CUtensorMapDataType type, int esize, const void *base,
                   uint64_t rows, uint64_t cols, uint32_t box_rows, uint32_t box_cols,
                   CUtensorMapSwizzle swz)
{
    EncodeFn enc = mx_encode_fn();
    if (!enc)
        return false;
    cuuint64_t gdim[2] = {cols, rows};
    cuuint64_t gstride[1] = {cols * uint64_t(esize)};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estride[2] = {1, 1};
    return enc(map, type, 2, const_cast<void *>(base), gdim, gstride, box, estride,
               CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <class Cfg>
static cudaError_t run_mx(const uint8_t *a, const uint8_t *sa, const uint8_t *b, const uint8_t *sb,
                          void *d, int64_t M, int64_t N, int64_t K, cudaStream_t stream, int num_sms)
{
    // scale-block arrays: [blocks][128 words of 4 bytes], one TMA box per block
    CUtensorMap tsa, tsb;
    const uint64_t KB = uint64_t(K / MX_BK);
    if (!mx_map(&tsa, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, sa, uint64_t(M / 128) * KB, 128, 1, 128,
                CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !mx_map(&tsb, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, sb, uint64_t(N / 128) * KB, 128, 1, 128,
                CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    auto kern = fp8_gemm_mx_kernel<Cfg>;
    // Per-device launch facts, worked out on the first launch of this configuration on
    // a device and cached: the shared-memory opt-in and (pair path) how many CTA pairs
    // fit on the GPU at once.
    static LaunchCache cache;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    int max_clusters = cache.get(dev);
    if (max_clusters == 0) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM);
        if (e != cudaSuccess)
            return e;
        max_clusters = 1;
        if (Cfg::CG == 2) {
            cudaLaunchConfig_t q = {};
            cudaLaunchAttribute qa[1];
            qa[0].id = cudaLaunchAttributeClusterDimension;
            qa[0].val.clusterDim.x = 2;
            qa[0].val.clusterDim.y = 1;
            qa[0].val.clusterDim.z = 1;
            q.blockDim = dim3(Cfg::THREADS);
            q.dynamicSmemBytes = Cfg::SMEM;
            q.attrs = qa;
            q.numAttrs = 1;
            q.gridDim = dim3(2 * unsigned(num_sms / 2));
            e = cudaOccupancyMaxActiveClusters(&max_clusters, kern, &q);
            if (e != cudaSuccess)
                return e;
            if (max_clusters < 1)
                return cudaErrorInvalidConfiguration;
        }
        cache.set(dev, max_clusters);
    }
    CUtensorMap ta, tb, td;
    const auto U8 = CU_TENSOR_MAP_DATA_TYPE_UINT8;
    if (!mx_map(&ta, U8, 1, a, uint64_t(M), uint64_t(K), MX_BM, MX_BK, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    const bool okb = (Cfg::MODE == 1)
                         ? mx_map(&tb, U8, 1, b, uint64_t(K), uint64_t(N), MX_BK, Cfg::B_BOX,
                                  CU_TENSOR_MAP_SWIZZLE_128B)  // W[K][N]
                         : mx_map(&tb, U8, 1, b, uint64_t(N), uint64_t(K), Cfg::B_ROWS, MX_BK,
                                  CU_TENSOR_MAP_SWIZZLE_128B);
    if (!okb)
        return cudaErrorInvalidValue;
    if (!mx_map(&td, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d, uint64_t(M), uint64_t(N), 32, 64,
                CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    const int64_t tiles = (M / Cfg::TILE_M) * (N / Cfg::BN);
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute at[2];
    set_pdl(at[0]);
    at[1].id = cudaLaunchAttributeClusterDimension;
    at[1].val.clusterDim.x = 2;
    at[1].val.clusterDim.y = 1;
    at[1].val.clusterDim.z = 1;
    cfg.blockDim = dim3(Cfg::THREADS);
    cfg.dynamicSmemBytes = Cfg::SMEM;
    cfg.stream = stream;
    cfg.attrs = at;
    if (Cfg::CG == 1) {
        cfg.numAttrs = 1;
        cfg.gridDim = dim3(unsigned(tiles < num_sms ? tiles : num_sms));
    } else {
        cfg.numAttrs = 2;
        const int64_t clusters = tiles < max_clusters ? tiles : max_clusters;
        cfg.gridDim = dim3(unsigned(2 * clusters));
    }
    e = cudaLaunchKernelEx(&cfg, kern, ta, tb, td, tsa, tsb, int(M), int(N), int(K));
    if (e != cudaSuccess)
        return e;
    return cudaGetLastError();
}

} // namespace

cudaError_t launch_gemm_mx(int mode, const uint8_t *a, const uint8_t *sa, const uint8_t *b,
                           const uint8_t *sb, void *d, int64_t M, int64_t N, int64_t K,
                           cudaStream_t stream, int num_sms)
{
    const bool pair = (M % 256) == 0 && (N % 256) == 0 && (M / 256) * (N / 256) >= 16;
    switch (mode) {
    case 0:
        return pair ? run_mx<MxCfg<256, 0, 2>>(a, sa, b, sb, d, M, N, K, stream, num_sms)
                    : run_mx<MxCfg<128, 0, 1>>(a, sa, b, sb, d, M, N, K, stream, num_sms);
    case 1:
        return pair ? run_mx<MxCfg<256, 1, 2>>(a, sa, b, sb, d, M, N, K, stream, num_sms)
                    : run_mx<MxCfg<128, 1, 1>>(a, sa, b, sb, d, M, N, K, stream, num_sms);
    default:
        return pair ? run_mx<MxCfg<256, 2, 2>>(a, sa, b, sb, d, M, N, K, stream, num_sms)
                    : run_mx<MxCfg<128, 2, 1>>(a, sa, b, sb, d, M, N, K, stream, num_sms);
    }
}

cudaError_t read_and_clear_mx_error(int *value)
{
    cudaError_t e = cudaMemcpyFromSymbol(value, g_mx_error, sizeof(int));
    if (e != cudaSuccess)
        return e;
    if (*value) {
        const int zero = 0;
        e = cudaMemcpyToSymbol(g_mx_error, &zero, sizeof(int));
    }
    return e;
}

} // namespace fp8bw
