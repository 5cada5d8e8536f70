// gemm.cu -- blockwise-scaled FP8 GEMM on the 5th-generation tensor cores (sm_100a).
//
// D[M][N] (BF16) = sum over 128-long reduction blocks kb of
//     (a-scale x b-scale of kb) * (sum_{k in kb} qa[m][k] * qb[n][k]),
// the fprop / dgrad / wgrad GEMMs of the FP8 linear layer (Puro-2B part 3/7,
// section 3.2: all three GEMMs use the FP8 path, with FP32 accumulation and a BF16
// result handed back to the model).
//
// Design (persistent, warp-specialised, one CTA per SM):
//   warp 0      TMA producer: per reduction block one 128x128 A tile and one B tile
//               (128B swizzle) into a STAGES-deep ring of shared-memory stages.
//   warp 1      MMA issuer: per reduction block 4 x tcgen05.mma kind::f8f6f4 (K = 32
//               bytes each) into one of two TMEM partial buffers (fresh accumulation
//               per block), then commits to the stage's "empty" barrier and to the
//               buffer's "full" barrier.
//   warp 2      scale loader: copies each reduction block's scales (a-scales of the
//               CTA's rows, b-scales of the tile) into a shared-memory ring with
//               cp.async, signalling a per-slot barrier when they land.
//   warp 3      idle (completes the first warpgroup, which gives registers away)
//   warps 4..11 promotion + epilogue: per block each thread loads its FP32 partial
//               from TMEM (one lane, i.e. row, and COLS columns in 64- or 32-column
//               loads; wgrad pairs: 4 rows x 32 columns per 16x256b load), releases
//               the buffer and adds partial x scale into an FP32 running sum in
//               registers (packed f32x2 FMA); last, it rounds to BF16 and stores.
// Double-buffered TMEM partials let the tensor cores run block kb+1 while the
// epilogue promotes block kb.
//
// CTA pairs (CG = 2, when M is a multiple of 256): a cluster of two CTAs computes a
// 256 x BN tile with tcgen05.mma.cta_group::2 issued by the even CTA.  Each CTA
// loads its own 128 rows of A and its own BN/2 columns of B (no multicast), and holds
// its 128 rows of D in its own TMEM, so per SM the shared-memory and L2 operand
// traffic per FLOP drops by a third against one CTA computing 128 x BN.
//
// Every wait is bounded (about one second); a wait that runs out records an error
// code in a device word and the whole CTA (pair) unwinds.
#include <cstdint>
#include <cstring>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "launch_cache.cuh"
#include "ptx.cuh"
#include "quant.cuh"

namespace fp8bw {

__device__ int g_device_error;  // first error code seen by a bounded wait (0 = none)

constexpr int BM = 128;  // rows of D per CTA
constexpr int BK = 128;  // one reduction block
constexpr uint64_t WAIT_LIMIT_NS = 1000000000ull;
constexpr uint64_t DRAIN_NS = 20000000ull;

enum : int { ERR_PRODUCER = 1, ERR_MMA_FULL = 2, ERR_MMA_TEMPTY = 3, ERR_EPI = 4, ERR_SCALES = 5 };

template <int BN_, int MODE_, int STAGES_, int CG_, bool OUT32_ = false>
struct GemmCfg {
    static constexpr int BN = BN_;      // columns of D per tile (both CTAs of a pair)
    static constexpr int MODE = MODE_;  // 0 fprop, 1 dgrad (B is MN-major), 2 wgrad
    static constexpr int STAGES = STAGES_;
    static constexpr int CG = CG_;      // CTAs per MMA (1 or 2)
    // OUT32: instead of storing BF16, add the FP32 sum into an FP32 output (wgrad
    // main-grad accumulation; TMA reduce-add on the pair path)
    static constexpr bool OUT32 = OUT32_;
    static constexpr int TILE_M = BM * CG;
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
    static constexpr int B_ROWS = BN / CG;  // B rows (N) this CTA loads per stage
    static constexpr int A_BYTES = BM * BK;
    static constexpr int B_BYTES = B_ROWS * BK;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    // TMEM holds NBUF partial buffers of BN fp32 columns (512 columns in all), so the
    // MMA can run NBUF-1 reduction blocks ahead of the promotion.
    static constexpr int NBUF = 512 / BN;
    static constexpr int TMEM_COLS = 512;
    // MN-major B (dgrad) boxes: 128 N-bytes with the 128-byte swizzle, or 64 with the
    // 64-byte swizzle when this CTA holds only 64 columns of B.
    static constexpr int B_BOX = (B_ROWS >= 128) ? 128 : 64;
    // Scale ring shared by the CTA, filled by the scale-loader warp: one slot per
    // (tile, reduction block) with the a-scales of the CTA's 128 rows and the
    // b-scale(s) of the tile: BN/128 block scales (fprop/dgrad) or BN column scales
    // (wgrad).
    static constexpr int SRING = 8;
    static constexpr int SB_FLOATS = (MODE == 2) ? BN : 4;
    static constexpr int SLOT_FLOATS = BM + SB_FLOATS;
    static constexpr int RING_BYTES = SRING * SLOT_FLOATS * 4;
    static_assert((SLOT_FLOATS * 4) % 16 == 0, "scale slots must stay 16-byte aligned");
    // Pair path: the finished tile leaves through shared memory and TMA bulk
    // stores; each epilogue warp owns 32 rows x COLS columns of BF16 staging, laid
    // out as 64-column boxes of 32 rows x 128 B with the 128-byte swizzle.
    static constexpr bool TMA_STORE = (CG == 2);
    // wgrad on the pair path promotes from the 16x256b TMEM layout (see the epilogue)
#ifndef FP8BW_WG16
#define FP8BW_WG16 1
#endif
    static constexpr bool WG16 = FP8BW_WG16 && MODE == 2 && TMA_STORE && COLS == 128;
    static_assert(!OUT32 || (MODE == 2 && (WG16 || !TMA_STORE)), "FP32 output is wgrad-only");
    static constexpr int STAGE_OUT_WARP = 32 * COLS * 2;
    static constexpr int OUT_BYTES = TMA_STORE ? EPI_WARPS * STAGE_OUT_WARP : 0;
    static constexpr int RING_OFF = STAGES * STAGE_BYTES + OUT_BYTES;
    static constexpr int BAR_OFF = RING_OFF + RING_BYTES;
    static constexpr int SMEM = 1024 + BAR_OFF + 512;
    static_assert(COLS % 32 == 0, "columns per thread must be whole TMEM load chunks");
    static_assert(BN % 128 == 0 && BN <= 256, "BN must be 128 or 256");
    static_assert(B_ROWS % B_BOX == 0, "B rows must be whole boxes");
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
                const __grid_constant__ CUtensorMap tmD, const float *__restrict__ sa, const float *__restrict__ sb,
                void *__restrict__ Dv, int M, int N, int K, int tiles_m, int KB)
{
    constexpr int BN = Cfg::BN, MODE = Cfg::MODE, STAGES = Cfg::STAGES, CG = Cfg::CG;
    constexpr int COLS = Cfg::COLS, EPI_WARPS = Cfg::EPI_WARPS;
    __nv_bfloat16 *D = static_cast<__nv_bfloat16 *>(Dv);
    float *D32 = static_cast<float *>(Dv);

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sout = smem + STAGES * Cfg::STAGE_BYTES;
    float *sring = reinterpret_cast<float *>(smem + Cfg::RING_OFF);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::BAR_OFF);
    uint64_t *full = bars;                 // [STAGES] TMA -> MMA   (used in the even CTA)
    uint64_t *empty = bars + STAGES;       // [STAGES] MMA -> TMA
    uint64_t *tfull = bars + 2 * STAGES;   // [NBUF] MMA -> epilogue
    uint64_t *tempty = tfull + Cfg::NBUF;  // [NBUF] epilogue -> MMA   (used in the even CTA)
    uint64_t *sfull = tempty + Cfg::NBUF;  // [SRING] scale loader -> epilogue
    uint64_t *sempty = sfull + Cfg::SRING; // [SRING] epilogue -> scale loader
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sempty + Cfg::SRING);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rank = (CG == 2) ? int(cluster_ctarank()) : 0;
    const int unit = (CG == 2) ? int(cluster_id_x()) : int(blockIdx.x);      // tile walker
    const int units = (CG == 2) ? int(cluster_count_x()) : int(gridDim.x);
    // A token count that is not a multiple of 128 (M for FPROP/DGRAD, K for WGRAD)
    // ends in a partial tile / reduction block: TMA reads zeros past the end of A and
    // B and clips the stores; the scale loader and the direct stores guard the rest.
    const int tiles_n = N / BN;  // tiles_m and KB (ceil divisions) come from the host
    const int num_tiles = tiles_m * tiles_n;


    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < Cfg::NBUF; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], EPI_WARPS * CG);
        }
        for (int r = 0; r < Cfg::SRING; ++r) {
            mbar_init(&sfull[r], 32);
            mbar_init(&sempty[r], EPI_WARPS);
        }
        *abort_flag = 0;
        fence_mbarrier_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    if (warp == 1) {
        tmem_alloc<CG>(tmem_slot, Cfg::TMEM_COLS);
        tmem_relinquish<CG>();
    }
    tc_fence_before();
    if (CG == 2)
        cluster_sync();  // barriers of both CTAs initialised before any remote arrive
    else
        __syncthreads();
    tc_fence_after();
    pdl_wait();               // inputs written by the previous kernel are visible
    pdl_launch_dependents();  // the next kernel may start its launch and prologue
    const uint32_t tmem_base = *tmem_slot;
    // cluster-window addresses of the even CTA's barriers
    const uint32_t full_lead = (CG == 2) ? mapa_shared(smem_u32(full), 0) : smem_u32(full);
    const uint32_t tempty_lead = (CG == 2) ? mapa_shared(smem_u32(tempty), 0) : smem_u32(tempty);

    if (warp < Cfg::EPI_WARP0) {
        regs_dec<Cfg::REGS_LOW>();
        if (warp == 0 && lane == 0) {
            // ---------------------------------------------------------- producer
            int stage = 0;
            uint32_t phase = 0;
            for (int t = unit; t < num_tiles && !*abort_flag; t += units) {
                int tm, tn;
                tile_coords(t, tiles_m, tiles_n, tm, tn);
                const int arow = tm * Cfg::TILE_M + rank * BM;
                const int bcol = tn * BN + rank * Cfg::B_ROWS;
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag, &g_device_error,
                                           ERR_PRODUCER, WAIT_LIMIT_NS))
                        goto role_done;
                    uint8_t *sA = smem + stage * Cfg::STAGE_BYTES;
                    uint8_t *sB = sA + Cfg::A_BYTES;
                    if (CG == 1) {
                        mbar_arrive_expect_tx(&full[stage], Cfg::STAGE_BYTES);
                        tma_load_2d(sA, &tmA, &full[stage], kb * BK, arow);
                        if (MODE == 1) {
                            // B = W[K][N] with N contiguous: boxes of B_BOX (N) x 128 (K).
#pragma unroll
                            for (int j = 0; j < Cfg::B_ROWS / Cfg::B_BOX; ++j)
                                tma_load_2d(sB + j * Cfg::B_BOX * BK, &tmB, &full[stage],
                                            bcol + j * Cfg::B_BOX, kb * BK);
                        } else {
                            tma_load_2d(sB, &tmB, &full[stage], kb * BK, bcol);
                        }
                    } else {
                        // The even CTA's barrier counts the bytes of both CTAs.
                        if (rank == 0)
                            mbar_arrive_expect_tx(&full[stage], 2 * Cfg::STAGE_BYTES);
                        const uint32_t fb = full_lead + uint32_t(stage) * 8u;
                        tma_load_2d_pair(sA, &tmA, fb, kb * BK, arow);
                        if (MODE == 1) {
#pragma unroll
                            for (int j = 0; j < Cfg::B_ROWS / Cfg::B_BOX; ++j)
                                tma_load_2d_pair(sB + j * Cfg::B_BOX * BK, &tmB, fb,
                                                 bcol + j * Cfg::B_BOX, kb * BK);
                        } else {
                            tma_load_2d_pair(sB, &tmB, fb, kb * BK, bcol);
                        }
                    }
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
        } else if (warp == 1 && lane == 0 && rank == 0) {
            // --------------------------------------------------------------- MMA
            constexpr uint32_t idesc = make_idesc_e4m3(Cfg::TILE_M, BN, MODE == 1 ? 1 : 0);
            int stage = 0, buf = 0;
            uint32_t phase = 0, tphase = 0;
            for (int t = unit; t < num_tiles && !*abort_flag; t += units) {
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_spin_bounded(&full[stage], phase, abort_flag, &g_device_error,
                                           ERR_MMA_FULL, WAIT_LIMIT_NS))
                        goto role_done;
                    if (!mbar_spin_bounded(&tempty[buf], tphase ^ 1u, abort_flag, &g_device_error,
                                           ERR_MMA_TEMPTY, WAIT_LIMIT_NS))
                        goto role_done;
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
                        if (MODE == 1 && Cfg::B_BOX == 128) {
                            // MN-major, 128B swizzle: 128 N-bytes per row, one row per k;
                            // atoms of 8 k-rows 1024 B apart (SBO), 128-wide N atoms
                            // 16 KB apart (LBO); a K step of 32 rows moves 4 KB.
                            bdesc = make_smem_desc_sw128(b_addr + k * 32 * 128, 128 * BK, 1024);
                        } else if (MODE == 1) {
                            // MN-major, 64B swizzle: 64 N-bytes per row; atoms of 8 k-rows
                            // 512 B apart (SBO); a K step of 32 rows moves 2 KB.
                            bdesc = make_smem_desc_sw64(b_addr + k * 32 * 64, 64 * BK, 512);
                        } else {
                            bdesc = make_smem_desc_sw128(b_addr + k * 32, 16, 1024);
                        }
                        mma_f8f6f4<CG>(d_tmem, adesc, bdesc, idesc, k > 0 ? 1u : 0u);
                    }
                    if (CG == 1) {
                        mma_commit(&empty[stage]);
                        mma_commit(&tfull[buf]);
                    } else {
                        mma_commit_pair(&empty[stage], 0x3);
                        mma_commit_pair(&tfull[buf], 0x3);
                    }
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                    if (++buf == Cfg::NBUF) {
                        buf = 0;
                        tphase ^= 1u;
                    }
                }
            }
        } else if (warp == 2) {
            // ------------------------------------------------------ scale loader
            // All 32 lanes copy one iteration's scales with cp.async; each lane's
            // copies arrive on the slot's "full" barrier when they land, so the warp
            // never waits for global memory and runs up to SRING iterations ahead.
            int j = 0;
            for (int t = unit; t < num_tiles && !*abort_flag; t += units) {
                int tm, tn;
                tile_coords(t, tiles_m, tiles_n, tm, tn);
                const float *sa_tile = sa + tm * Cfg::TILE_M + rank * BM;
                const int nb0 = (tn * BN) / 128;
                for (int kb = 0; kb < KB; ++kb, ++j) {
                    const int r = j % Cfg::SRING;
                    const uint32_t ph = uint32_t(j / Cfg::SRING) & 1u;
                    const bool ok = mbar_wait_bounded(&sempty[r], ph ^ 1u, abort_flag,
                                                      &g_device_error, ERR_SCALES, WAIT_LIMIT_NS);
                    if (!__all_sync(0xffffffffu, ok))
                        goto role_done;
                    float *slot = sring + r * Cfg::SLOT_FLOATS;
                    if (MODE == 2) {  // the CTA's 128 row scales (M is a feature count)
                        cp_async_16(slot + 4 * lane, sa_tile + size_t(kb) * M + 4 * lane);
                    } else {  // M counts tokens: rows past M (a partial tile) read as zeros
                        const int row = tm * Cfg::TILE_M + rank * BM + 4 * lane;
                        cp_async_16_zfill(slot + 4 * lane,
                                          row < M ? sa_tile + size_t(kb) * M + 4 * lane : sa,
                                          row < M);
                    }
                    if (MODE == 0) {
                        if (lane < BN / 128)
                            cp_async_4(slot + BM + lane, sb + size_t(nb0 + lane) * KB + kb);
                    } else if (MODE == 1) {
                        if (lane < BN / 128)
                            cp_async_4(slot + BM + lane, sb + size_t(kb) * (N / 128) + nb0 + lane);
                    } else if (Cfg::WG16) {
                        // Column scales in the order the 16x256b promotion reads them:
                        // column 128 h + 64 cc + 8 j + 2 t0 + e goes to slot position
                        // 128 h + 64 cc + 16 t0 + 2 j + e, so a thread's 16 scales of one
                        // 64-column chunk are contiguous (four 16-byte loads).  Lane l copies
                        // columns 8 l .. 8 l + 7 (j = l % 8) as four 8-byte pieces.
                        const float *src = sb + size_t(kb) * N + tn * BN + lane * 8;
                        float *dst = slot + BM + (lane >> 3) * 64 + (lane & 7) * 2;
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            cp_async_8(dst + 16 * q, src + 2 * q);
                    } else {
                        const float *src = sb + size_t(kb) * N + tn * BN + lane * (BN / 32);
#pragma unroll
                        for (int q = 0; q < BN / 128; ++q)
                            cp_async_16(slot + BM + lane * (BN / 32) + 4 * q, src + 4 * q);
                    }
                    cp_async_mbar_arrive(&sfull[r]);
                }
            }
            cp_async_wait<0>();
        }
    role_done:;
    } else {
        regs_inc<Cfg::REGS_HIGH>();
        // ---------------------------------------------------- promotion + epilogue
        const int ew = warp - Cfg::EPI_WARP0;
        const int quarter = warp & 3;           // TMEM lanes this warp may access
        const int col0 = (ew >> 2) * COLS;      // columns of the tile this thread owns
        const int row_in_tile = rank * BM + quarter * 32 + lane;

        const int row_local = quarter * 32 + lane;  // the thread's row among the CTA's 128

        float2 acc[COLS / 2];
#pragma unroll
        for (int i = 0; i < COLS / 2; ++i)
            acc[i] = make_float2(0.f, 0.f);

        const int my_tiles = (num_tiles - unit + units - 1) / units;
        const int total_iters = my_tiles > 0 ? my_tiles * KB : 0;

        int buf = 0, kb = 0, t = unit, tm = 0, tn = 0;
        uint32_t tphase = 0;
        tile_coords(t, tiles_m, tiles_n, tm, tn);
        for (int j = 0; j < total_iters; ++j) {
            const int r = j % Cfg::SRING;
            const bool sready = mbar_wait_bounded(&sfull[r], uint32_t(j / Cfg::SRING) & 1u,
                                                  abort_flag, &g_device_error, ERR_SCALES,
                                                  WAIT_LIMIT_NS);
            const float *slot = sring + r * Cfg::SLOT_FLOATS;
            // busy-poll: this handshake is on the critical path of every block
            const bool ready = sready && mbar_spin_bounded(&tfull[buf], tphase, abort_flag,
                                                           &g_device_error, ERR_EPI,
                                                           WAIT_LIMIT_NS);
            if (!__all_sync(0xffffffffu, ready))  // leave together: tcgen05.ld is warp-wide
                break;
            tc_fence_after();
            const float a_s = slot[row_local];
            const uint32_t taddr =
                tmem_base + (uint32_t(quarter * 32) << 16) + uint32_t(buf * BN + col0);
            const float sc = (MODE == 2) ? a_s : a_s * slot[BM + col0 / 128];
            const float2 sc2 = make_float2(sc, sc);

            if constexpr (Cfg::WG16) {
                // wgrad, 16x256b layout: thread (t0, t1) = (lane % 4, lane / 4) holds
                // rows t1 + 8i (i < 4) of the warp's 32 and columns 64cc + 8j + 2t0 + {0,1}
                // (cc < 2, j < 8) of its 128, so each column-scale pair read from shared
                // memory serves four rows.
                const int t0 = lane & 3, t1 = lane >> 2;
                float2 sa2[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float v = slot[quarter * 32 + t1 + 8 * i];
                    sa2[i] = make_float2(v, v);
                }
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    float2 sbp[8];
                    {
                        // this thread's 16 column scales of chunk cc, contiguous (see the
                        // scale loader)
                        const float4 *sp =
                            reinterpret_cast<const float4 *>(slot + BM + col0 + 64 * cc + 16 * t0);
#pragma unroll
                        for (int m = 0; m < 4; ++m) {
                            const float4 v = sp[m];
                            sbp[2 * m] = make_float2(v.x, v.y);
                            sbp[2 * m + 1] = make_float2(v.z, v.w);
                        }
                    }
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        uint32_t v[32];
                        tmem_ld_16x256b_x8(taddr + (uint32_t(16 * h) << 16) + uint32_t(64 * cc), v);
                        tmem_wait_ld();
                        if (cc == 1 && h == 1) {
                            tc_fence_before();
                            __syncwarp();
                            if (lane == 0) {
                                if (CG == 1 || rank == 0)
                                    mbar_arrive(&tempty[buf]);
                                else
                                    mbar_arrive_cluster(tempty_lead + uint32_t(buf) * 8u);
                            }
                        }
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
#pragma unroll
                            for (int e = 0; e < 2; ++e) {
                                const int i = 2 * h + e;
                                const float2 p = make_float2(__uint_as_float(v[4 * j + 2 * e]),
                                                             __uint_as_float(v[4 * j + 2 * e + 1]));
                                float2 &a = acc[i * 16 + cc * 8 + j];
                                a = __ffma2_rn(__fmul2_rn(p, sbp[j]), sa2[i], a);
                            }
                        }
                    }
                }
            } else {
                // TMEM -> registers in chunks of CW columns (GRP of them before one
                // wait): 64-column loads where the thread's columns allow (fewer, larger
                // tcgen05.ld per block; measured 1-4% faster than 32-column ones).  The
                // buffer goes back to the MMA as soon as the last chunk is in registers.
                constexpr int CW = (COLS % 64 == 0) ? 64 : 32;
                constexpr int CHUNKS = COLS / CW;
                constexpr int GRP = (CW == 64) ? 1 : ((CHUNKS <= 2) ? CHUNKS : 1);
    #pragma unroll
                for (int cg = 0; cg < CHUNKS; cg += GRP) {
                    uint32_t v[GRP][CW];
    #pragma unroll
                    for (int g = 0; g < GRP; ++g) {
                        if constexpr (CW == 64)
                            tmem_ld_32x32b_x64(taddr + uint32_t((cg + g) * CW), v[g]);
                        else
                            tmem_ld_32x32b_x32(taddr + uint32_t((cg + g) * CW), v[g]);
                    }
                    tmem_wait_ld();
                    if (cg + GRP == CHUNKS) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) {
                            if (CG == 1 || rank == 0)
                                mbar_arrive(&tempty[buf]);
                            else  // the MMA issuer lives in the even CTA
                                mbar_arrive_cluster(tempty_lead + uint32_t(buf) * 8u);
                        }
                    }
    #pragma unroll
                    for (int g = 0; g < GRP; ++g) {
                        const int c = cg + g;
    #pragma unroll
                        for (int jj = 0; jj < CW / 2; jj += 2) {
                            const float2 p0 = make_float2(__uint_as_float(v[g][2 * jj]),
                                                          __uint_as_float(v[g][2 * jj + 1]));
                            const float2 p1 = make_float2(__uint_as_float(v[g][2 * jj + 2]),
                                                          __uint_as_float(v[g][2 * jj + 3]));
                            float2 &a0 = acc[c * (CW / 2) + jj];
                            float2 &a1 = acc[c * (CW / 2) + jj + 1];
                            if (MODE == 2) {
                                const float4 bs = *reinterpret_cast<const float4 *>(
                                    slot + BM + col0 + c * CW + 2 * jj);
                                a0 = __ffma2_rn(__fmul2_rn(p0, make_float2(bs.x, bs.y)), sc2, a0);
                                a1 = __ffma2_rn(__fmul2_rn(p1, make_float2(bs.z, bs.w)), sc2, a1);
                            } else {
                                a0 = __ffma2_rn(p0, sc2, a0);
                                a1 = __ffma2_rn(p1, sc2, a1);
                            }
                        }
                    }
                }
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&sempty[r]);  // this warp is done with the slot's scales
            if (++kb == KB) {
                if constexpr (Cfg::OUT32 && Cfg::TMA_STORE) {
                    // FP32 tile -> swizzled staging (32 rows x 64 columns per pass, two
                    // 32x32 boxes) -> bulk tensor reduce-add into the FP32 output.
                    uint8_t *stg = sout + ew * Cfg::STAGE_OUT_WARP;
                    const int t0 = lane & 3, t1 = lane >> 2;
                    const int r0 = tm * Cfg::TILE_M + rank * BM + quarter * 32;
#pragma unroll
                    for (int cc = 0; cc < 2; ++cc) {
                        if (lane == 0)
                            bulk_wait_read0();
                        __syncwarp();
#pragma unroll
                        for (int i = 0; i < 4; ++i)
#pragma unroll
                            for (int j = 0; j < 8; ++j) {
                                const int row = t1 + 8 * i;
                                const int chunk = 2 * (j & 3) + (t0 >> 1);
                                *reinterpret_cast<float2 *>(stg + (j >> 2) * 4096 + row * 128 +
                                                            ((chunk ^ (row & 7)) << 4) +
                                                            8 * (t0 & 1)) =
                                    acc[i * 16 + cc * 8 + j];
                            }
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            tma_reduce_add_2d(&tmD, stg, tn * BN + col0 + 64 * cc, r0);
                            tma_reduce_add_2d(&tmD, stg + 4096, tn * BN + col0 + 64 * cc + 32, r0);
                            bulk_commit();
                        }
                    }
                } else if constexpr (Cfg::OUT32) {
                    // Vector atomic adds (red.global.add.v4.f32): calls that overlap on the
                    // same FP32 buffer only reorder their additions, as on the pair path.
                    float *dst = D32 + size_t(tm * Cfg::TILE_M + row_in_tile) * size_t(N) +
                                 size_t(tn * BN + col0);
#pragma unroll
                    for (int c = 0; c < COLS / 4; ++c)
                        atomicAdd(reinterpret_cast<float4 *>(dst + 4 * c),
                                  make_float4(acc[2 * c].x, acc[2 * c].y, acc[2 * c + 1].x,
                                              acc[2 * c + 1].y));
                } else if (Cfg::TMA_STORE) {
                    // BF16 tile -> swizzled staging -> two bulk tensor stores per warp.
                    uint8_t *stg = sout + ew * Cfg::STAGE_OUT_WARP;
                    if (lane == 0)
                        bulk_wait_read0();  // the previous tile's stores have read it
                    __syncwarp();
                    if constexpr (Cfg::WG16) {
                        // rows t1 + 8i, columns 64cc + 8j + 2t0: one 4-byte store each,
                        // into chunk j of box cc (conflict-free under the swizzle)
                        const int t0 = lane & 3, t1 = lane >> 2;
#pragma unroll
                        for (int i = 0; i < 4; ++i)
#pragma unroll
                            for (int cc = 0; cc < 2; ++cc)
#pragma unroll
                                for (int j = 0; j < 8; ++j) {
                                    const int row = t1 + 8 * i;
                                    __nv_bfloat162 h =
                                        __float22bfloat162_rn(acc[i * 16 + cc * 8 + j]);
                                    *reinterpret_cast<uint32_t *>(
                                        stg + cc * 4096 + row * 128 + ((j ^ (row & 7)) << 4) +
                                        4 * t0) = *reinterpret_cast<uint32_t *>(&h);
                                }
                    } else {
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
                        const int box = c >> 3, chunk = c & 7;
                        *reinterpret_cast<uint4 *>(stg + box * 4096 + lane * 128 +
                                                   ((chunk ^ (lane & 7)) << 4)) = o;
                    }
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        const int r0 = tm * Cfg::TILE_M + rank * BM + quarter * 32;
#pragma unroll
                        for (int box = 0; box < COLS / 64; ++box)
                            tma_store_2d(&tmD, stg + box * 4096, tn * BN + col0 + box * 64, r0);
                        bulk_commit();
                    }
                } else {
                    __nv_bfloat16 *dst = D + size_t(tm * Cfg::TILE_M + row_in_tile) * size_t(N) +
                                         size_t(tn * BN + col0);
                    if (tm * Cfg::TILE_M + row_in_tile < M) {  // rows past M: not stored
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
                    }
                }
#pragma unroll
                for (int q = 0; q < COLS / 2; ++q)
                    acc[q] = make_float2(0.f, 0.f);
                kb = 0;
                t += units;
                if (t < num_tiles)
                    tile_coords(t, tiles_m, tiles_n, tm, tn);
            }
            if (++buf == Cfg::NBUF) {
                buf = 0;
                tphase ^= 1u;
            }
        }
        if (Cfg::TMA_STORE && lane == 0)
            bulk_wait0();  // output stores complete before the CTA leaves
    }

    tc_fence_before();
    __syncthreads();
    if (*abort_flag && threadIdx.x == 0) {
        // Unwind after a wait ran out: give copies and MMAs still in flight time to
        // land before the CTA's shared and tensor memory are released.
        const uint64_t t0 = global_timer_ns();
        while (global_timer_ns() - t0 < DRAIN_NS) {
        }
    }
    if (CG == 2)
        cluster_sync();  // the partner no longer reads this CTA's memory or barriers
    else
        __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc<CG>(tmem_base, Cfg::TMEM_COLS);
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

// 2-D uint8 tensor map over a row-major [rows][cols] array, box {box_cols, box_rows}.
static bool make_map_u8(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols,
                        uint32_t box_rows, uint32_t box_cols,
                        CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B)
{
    EncodeTiledFn enc = get_encode_fn();
    if (!enc)
        return false;
    cuuint64_t gdim[2] = {cols, rows};
    cuuint64_t gstride[1] = {cols};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estride[2] = {1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), gdim, gstride,
                     box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// BF16 [rows][cols] output map for TMA stores: box 64 columns (128 B) x 32 rows,
// 128-byte swizzle.
static bool make_map_bf16_out(CUtensorMap *map, void *base, uint64_t rows, uint64_t cols)
{
    EncodeTiledFn enc = get_encode_fn();
    if (!enc)
        return false;
    cuuint64_t gdim[2] = {cols, rows};
    cuuint64_t gstride[1] = {cols * 2};
    cuuint32_t box[2] = {64, 32};
    cuuint32_t estride[2] = {1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, gdim, gstride, box, estride,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// FP32 [rows][cols] output map for TMA reduce-add: box 32 columns (128 B) x 32 rows,
// 128-byte swizzle.
static bool make_map_f32_out(CUtensorMap *map, void *base, uint64_t rows, uint64_t cols)
{
    EncodeTiledFn enc = get_encode_fn();
    if (!enc)
        return false;
    cuuint64_t gdim[2] = {cols, rows};
    cuuint64_t gstride[1] = {cols * 4};
    cuuint32_t box[2] = {32, 32};
    cuuint32_t estride[2] = {1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, base, gdim, gstride, box, estride,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <class Cfg>
static cudaError_t run(const uint8_t *a, const float *sa, const uint8_t *b, const float *sb,
                       void *d, int64_t M, int64_t N, int64_t K, cudaStream_t stream, int num_sms)
{
    auto kern = fp8_gemm_kernel<Cfg>;
    // Per-device launch facts, worked out on the first launch of this configuration on
    // a device and cached: the register-split check, the shared-memory opt-in and (pair
    // path) how many CTA pairs fit on the GPU at once.
    static LaunchCache cache;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    int max_clusters = cache.get(dev);
    if (max_clusters == 0) {
        cudaFuncAttributes attr;
        e = cudaFuncGetAttributes(&attr, kern);
        if (e != cudaSuccess)
            return e;
        // setmaxnreg.inc waits until enough registers are free; refuse to launch a
        // split the launch allocation cannot cover (it would never make progress).
        if (attr.numRegs * Cfg::THREADS < Cfg::REGS_NEEDED)
            return cudaErrorInvalidConfiguration;
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
    CUtensorMap ta, tb;
    if (!make_map_u8(&ta, a, uint64_t(M), uint64_t(K), BM, BK))
        return cudaErrorInvalidValue;
    bool ok;
    if (Cfg::MODE == 1)
        ok = make_map_u8(&tb, b, uint64_t(K), uint64_t(N), BK, Cfg::B_BOX,  // W[K][N]
                         Cfg::B_BOX == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B);
    else
        ok = make_map_u8(&tb, b, uint64_t(N), uint64_t(K), Cfg::B_ROWS, BK);
    if (!ok)
        return cudaErrorInvalidValue;
    CUtensorMap td;
    std::memset(&td, 0, sizeof td);
    if (Cfg::TMA_STORE && !Cfg::OUT32 && !make_map_bf16_out(&td, d, uint64_t(M), uint64_t(N)))
        return cudaErrorInvalidValue;
    if (Cfg::TMA_STORE && Cfg::OUT32 && !make_map_f32_out(&td, d, uint64_t(M), uint64_t(N)))
        return cudaErrorInvalidValue;
    const int64_t tiles = ((M + Cfg::TILE_M - 1) / Cfg::TILE_M) * (N / Cfg::BN);
    void *dp = d;
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
    e = cudaLaunchKernelEx(&cfg, kern, ta, tb, td, sa, sb, dp, int(M), int(N), int(K),
                           int((M + Cfg::TILE_M - 1) / Cfg::TILE_M), int((K + BK - 1) / BK));
    if (e != cudaSuccess)
        return e;
    return cudaGetLastError();
}

#ifndef FP8BW_PAIR
#define FP8BW_PAIR 1
#endif
#ifndef FP8BW_PAIR_BN
#define FP8BW_PAIR_BN 256
#endif

cudaError_t launch_gemm(int mode, const uint8_t *a, const float *sa, const uint8_t *b,
                        const float *sb, void *d, int64_t M, int64_t N, int64_t K,
                        cudaStream_t stream, int num_sms)
{
    constexpr int PBN = FP8BW_PAIR_BN;                 // N of a pair tile
    constexpr int PST = (PBN == 256) ? 4 : 6;          // pair-path pipeline stages
    // Single-CTA path: 128-wide tiles when N is not a multiple of 256, and also when
    // 256-wide ones would leave most SMs idle (fewer tiles than half the SMs, e.g. the
    // 128 x 1024 x 1024 single-layer fprop: 4 tiles of 128 x 256 or 8 of 128 x 128).
    const bool wide = (N % 256) == 0 && ((M + 127) / 128) * (N / 256) * 2 >= num_sms;
    const bool pair = FP8BW_PAIR && (N % PBN) == 0 && (M % 256) == 0 &&
                      (M / 256) * (N / PBN) >= 16;
    switch (mode) {
    case 0:
        if (pair)
            return run<GemmCfg<PBN, 0, PST, 2>>(a, sa, b, sb, d, M, N, K, stream, num_sms);
        return wide ? run<GemmCfg<256, 0, 4, 1>>(a, sa, b, sb, d, M, N, K, stream, num_sms)
                    : run<GemmCfg<128, 0, 6, 1>>(a, sa, b, sb, d, M, N, K, stream, num_sms);
    case 1:
        if (pair)
            return run<GemmCfg<PBN, 1, PST, 2>>(a, sa, b, sb, d, M, N, K, stream, num_sms);
        return wide ? run<GemmCfg<256, 1, 4, 1>>(a, sa, b, sb, d, M, N, K, stream, num_sms)
                    : run<GemmCfg<128, 1, 6, 1>>(a, sa, b, sb, d, M, N, K, stream, num_sms);
    default:
        if (pair)
            return run<GemmCfg<PBN, 2, PST, 2>>(a, sa, b, sb, d, M, N, K, stream, num_sms);
        return wide ? run<GemmCfg<256, 2, 4, 1>>(a, sa, b, sb, d, M, N, K, stream, num_sms)
                    : run<GemmCfg<128, 2, 6, 1>>(a, sa, b, sb, d, M, N, K, stream, num_sms);
    }
}

cudaError_t launch_gemm_wgrad_acc32(const uint8_t *a, const float *sa, const uint8_t *b,
                                    const float *sb, float *d32, int64_t M, int64_t N, int64_t K,
                                    cudaStream_t stream, int num_sms)
{
    const bool wide = (N % 256) == 0;
    const bool pair = FP8BW_PAIR && FP8BW_WG16 && wide && (M % 256) == 0 &&
                      (M / 256) * (N / 256) >= 16;
    if (pair)
        return run<GemmCfg<256, 2, 4, 2, true>>(a, sa, b, sb, d32, M, N, K, stream, num_sms);
    return wide ? run<GemmCfg<256, 2, 4, 1, true>>(a, sa, b, sb, d32, M, N, K, stream, num_sms)
                : run<GemmCfg<128, 2, 6, 1, true>>(a, sa, b, sb, d32, M, N, K, stream, num_sms);
}

// Self-test of the bounded-wait path: one warp waits, with the same bounded wait the
// GEMM uses, on a shared-memory barrier that nothing ever arrives on.  The wait runs
// out after limit_ns, records ERR_SELFTEST in the device error word and the kernel
// returns normally; no fault, trap or unbounded wait is involved.
enum : int { ERR_SELFTEST = 7 };

__global__ void __launch_bounds__(32) selftest_wait_kernel(uint64_t limit_ns)
{
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbarrier_init();
    }
    __syncwarp();
    if (threadIdx.x == 0)
        mbar_wait_bounded(&bar, 0u, &abort_flag, &g_device_error, ERR_SELFTEST, limit_ns);
    __syncwarp();
}

cudaError_t launch_selftest_wait(uint64_t limit_ns, cudaStream_t stream)
{
    selftest_wait_kernel<<<1, 32, 0, stream>>>(limit_ns);
    return cudaGetLastError();
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
