// Cluster and CTA-pair helpers of the two-SM prefill kernels (sm_100a):
// cluster ranks and shared::cluster addresses, TMA loads that complete on the
// leader CTA's mbarrier, and the tcgen05 operations of a CTA pair
// (.cta_group::2: tensor-memory allocation, M = 256 MMAs, commits that
// arrive in both CTAs).  No copy here multicasts.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "patch_common.cuh"

namespace patchk {

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// shared::cluster address of the same shared-memory offset in CTA `rank`
__device__ __forceinline__ uint32_t map_to_rank(const void *p, uint32_t rank) {
    uint32_t out;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(out) : "r"(smem_u32(p)), "r"(rank));
    return out;
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void fence_mbar_init_cluster() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
                 : "memory");
}
__device__ __forceinline__ void st_cluster_u32(uint32_t cluster_addr, uint32_t v) {
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(cluster_addr), "r"(v) : "memory");
}
// 2-D / 3-D TMA loads into this CTA's shared memory, completing on an
// mbarrier that may live in the peer CTA (cluster address)
__device__ __forceinline__ void tma2d_pair(void *dst, const void *tmap, int32_t x, int32_t y,
                                           uint32_t mbar_cluster) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
        "l"(tmap), "r"(x), "r"(y), "r"(mbar_cluster)
        : "memory");
}
__device__ __forceinline__ void tma3d_pair(void *dst, const void *tmap, int32_t x, int32_t y, int32_t z,
                                           uint32_t mbar_cluster) {
    asm volatile(
        "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
        "l"(tmap), "r"(x), "r"(y), "r"(z), "r"(mbar_cluster)
        : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t *slot, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
// commit: arrive on the mbarrier at this offset in both CTAs of the pair
// once every tcgen05 operation issued so far has completed
__device__ __forceinline__ void tc_commit_pair(uint64_t *bar) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
            smem_u32(bar)),
        "h"(static_cast<uint16_t>(3))
        : "memory");
}
__device__ __forceinline__ void mma_dense_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                               uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void mma_sparse_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                                uint32_t e_tmem, uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %5, 0;\n\t"
        "tcgen05.mma.sp.cta_group::2.kind::f16 [%0], %1, %2, [%3], %4, p;\n\t}\n" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(e_tmem), "r"(idesc), "r"(accumulate)
        : "memory");
}
// One k-step of MMAs back to back in one asm block (descriptors computed up
// front): four dense M256 K16 MMAs, or two 2:4 M256 K32 MMAs with metadata
// selectors 0 and 1.  `accumulate` applies to the first MMA; the others
// always accumulate.
__device__ __forceinline__ void mma_dense_pair_x4(uint32_t d_tmem, uint64_t a0, uint64_t a1, uint64_t a2,
                                                  uint64_t a3, uint64_t b0, uint64_t b1, uint64_t b2, uint64_t b3,
                                                  uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p, t;\n\t"
        "setp.ne.b32 p, %10, 0;\n\t"
        "setp.eq.b32 t, %9, %9;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %5, %9, p;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %2, %6, %9, t;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %3, %7, %9, t;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %4, %8, %9, t;\n\t}\n" ::"r"(d_tmem),
        "l"(a0), "l"(a1), "l"(a2), "l"(a3), "l"(b0), "l"(b1), "l"(b2), "l"(b3), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void mma_sparse_pair_x2(uint32_t d_tmem, uint64_t a0, uint64_t a1, uint64_t b0,
                                                   uint64_t b1, uint32_t e_tmem, uint32_t idesc0, uint32_t idesc1,
                                                   uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p, t;\n\t"
        "setp.ne.b32 p, %8, 0;\n\t"
        "setp.eq.b32 t, %6, %6;\n\t"
        "tcgen05.mma.sp.cta_group::2.kind::f16 [%0], %1, %3, [%5], %6, p;\n\t"
        "tcgen05.mma.sp.cta_group::2.kind::f16 [%0], %2, %4, [%5], %7, t;\n\t}\n" ::"r"(d_tmem),
        "l"(a0), "l"(a1), "l"(b0), "l"(b1), "r"(e_tmem), "r"(idesc0), "r"(idesc1), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void tmem_cp_pair_128x128b(uint32_t taddr, uint64_t s_desc) {
    asm volatile("tcgen05.cp.cta_group::2.128x128b [%0], %1;" ::"r"(taddr), "l"(s_desc) : "memory");
}
// instruction descriptor: bf16 x bf16 -> fp32, K-major A and B, M = 256
__host__ __device__ constexpr uint32_t idesc_pair(int n, bool sparse, uint32_t id2 = 0) {
    return (id2 & 3u) | (sparse ? (1u << 2) : 0u) | (1u << 4) | (1u << 7) | (1u << 10) |
           (static_cast<uint32_t>(n >> 3) << 17) | (static_cast<uint32_t>(256 >> 4) << 24);
}

}  // namespace patchk
