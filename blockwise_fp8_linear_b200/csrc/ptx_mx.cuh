// ptx_mx.cuh -- inline-PTX wrappers for the block-scaled (E8M0) tcgen05 GEMM: the
// block-scaled MMA, shared-memory -> tensor-memory copies of scale factors, and the
// descriptors and fences they need.  Builds on ptx.cuh.
#pragma once
#include <cstdint>

#include "ptx.cuh"

namespace fp8bw {

// ----------------------------------------------- block-scaled MMA (E8M0 scales)

// Instruction descriptor for kind::mxf8f6f4.block_scale, E4M3 x E4M3 -> F32 with E8M0
// scale factors (the block-scaled descriptor has no D-format field):
//   bits 4-5 B scale-factor byte   bits 7-9 / 10-12 A / B format (0 = E4M3)
//   bit 16 B major                 bits 17-22 N >> 3     bit 23 scale format (1 = E8M0)
//   bits 24-28 M >> 4              bits 29-30 A scale-factor byte
__host__ __device__ constexpr uint32_t make_idesc_mx_e4m3(int m, int n, int b_mn_major, int sf_id)
{
    return ((uint32_t)sf_id << 4) | ((uint32_t)b_mn_major << 16) | ((uint32_t)(n >> 3) << 17) |
           (1u << 23) | ((uint32_t)(m >> 4) << 24) | ((uint32_t)sf_id << 29);
}

// D (+)= A x B with per-32-K E8M0 scale factors read from tensor memory: sfa / sfb are
// TMEM addresses whose top two bits select the byte of each 32-bit scale word.
template <int CG>
__device__ __forceinline__ void mma_mxf8f6f4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                             uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                             uint32_t accumulate)
{
    if (CG == 1)
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
            ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
            : "memory");
    else
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
            ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
            : "memory");
}

// Shared memory -> tensor memory: 32 rows x 128 bits from shared memory, written to
// TMEM lanes 0-31 (4 columns) and repeated in the other three 32-lane quarters.
// With cta_group::2, issued by the even CTA, each CTA of the pair copies from its own
// shared memory into its own tensor memory.
template <int CG>
__device__ __forceinline__ void tmem_cp_32x128b_warpx4(uint32_t taddr, uint64_t src_desc)
{
    if (CG == 1)
        asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(src_desc)
                     : "memory");
    else
        asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(src_desc)
                     : "memory");
}

// Descriptor of a no-swizzle, K-major shared-memory region of 16-byte rows (core
// matrices of 8 rows x 16 bytes, 128 bytes apart): the source of tcgen05.cp.
__device__ __forceinline__ uint64_t make_smem_desc_rows16(uint32_t saddr)
{
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)1 << 16;                 // 16 bytes (unused: one 16-byte column)
    d |= (uint64_t)(128 >> 4) << 32;        // next 8 rows
    d |= (uint64_t)1 << 46;                 // version
    return d;                               // layout type 0: no swizzle
}

// Generic-proxy shared-memory writes made visible to the async proxy (tcgen05.cp).
__device__ __forceinline__ void fence_proxy_async_all()
{
    asm volatile("fence.proxy.async;" ::: "memory");
}

// Arrive on an mbarrier of the peer CTA, releasing this thread's prior writes at
// cluster scope.
__device__ __forceinline__ void mbar_arrive_cluster_release(uint32_t cluster_addr)
{
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
                 : "memory");
}

// 16-byte store into the shared memory of a CTA of the cluster (cluster-window address).
__device__ __forceinline__ void st_shared_cluster_v4(uint32_t cluster_addr, uint4 v)
{
    asm volatile("st.shared::cluster.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(cluster_addr), "r"(v.x),
                 "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

// Generic-proxy writes to any CTA's shared memory of the cluster made visible to the
// async proxy (tcgen05.cp of a CTA pair reads both CTAs' shared memory).
__device__ __forceinline__ void fence_proxy_async_cluster()
{
    asm volatile("fence.proxy.async.shared::cluster;" ::: "memory");
}

} // namespace fp8bw
