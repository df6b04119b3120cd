// gdla_pair.cuh - PTX wrappers for CTA pairs (a cluster of two CTAs running
// tcgen05 MMAs with cta_group::2), sm_100a.
//
// A pair's M = 256 MMA is issued by the even CTA: each CTA holds its own 128 rows of
// A (and of D in its TMEM) and half of B's N rows at the same shared-memory offset.
// Both CTAs' TMA loads complete on the even CTA's mbarrier; MMA completion is
// signalled to both CTAs by one commit.
#pragma once

#include "gdla_ptx.cuh"

namespace gdla {

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Shared::cluster address of the same offset in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}
// Arrive on an mbarrier given by its shared::cluster address (possibly the peer's).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
// Bounded wait (as mbar_wait) with cluster-scope acquire, for barriers that the
// peer CTA's threads, its TMA loads or the pair's MMAs arrive on.
__device__ __forceinline__ bool mbar_wait_cl(uint64_t *bar, uint32_t parity, volatile int *abort, int site) {
    const uint32_t a = smem_u32(bar);
    if (mbar_try_wait_cluster(a, parity)) return true;
    const long long start = clock64();
    while (true) {
        for (int i = 0; i < 64; ++i)
            if (mbar_try_wait_cluster(a, parity)) return true;
        if (*abort) return false;
        if (clock64() - start > kWaitLimitCycles) {
            *abort = 1;
            atomicExch(&g_device_error, site);
            return false;
        }
    }
}
// Wait at most `cycles` for a phase (cluster scope), ignoring the abort flag.
__device__ __forceinline__ bool mbar_wait_cl_cycles(uint64_t *bar, uint32_t parity, long long cycles) {
    const uint32_t a = smem_u32(bar);
    const long long start = clock64();
    while (!mbar_try_wait_cluster(a, parity))
        if (clock64() - start > cycles) return false;
    return true;
}
// TMA load into this CTA's shared memory whose completion is counted on the even
// CTA's mbarrier: `bar` is this CTA's copy; clearing the peer bit of its
// shared::cluster address selects the even CTA's.
constexpr uint32_t kPeerBitMask = 0xFEFFFFFFu;
__device__ __forceinline__ void tma_load_3d_pair(void *dst, const CUtensorMap *map, uint64_t *bar, int c0, int c1,
                                                 int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar) & kPeerBitMask), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}
// TMEM allocation of a pair: one warp with the same warp index in each CTA.
__device__ __forceinline__ void tmem_alloc_pair(uint32_t *dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void umma_ss_pair_leader(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                                    uint32_t accumulate, uint32_t leader) {
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "setp.ne.b32 q, %5, 0;\n\t"
        "@q tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(leader)
        : "memory");
}
// Arrive once on `bar` (same offset) in both CTAs of the pair when the pair's MMAs
// issued so far are done.
__device__ __forceinline__ void umma_commit_pair_leader(uint64_t *bar, uint32_t leader) {
    asm volatile(
        "{\n\t.reg .pred q;\n\t"
        "setp.ne.b32 q, %1, 0;\n\t"
        "@q tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %2;\n\t}" ::"r"(
            smem_u32(bar)),
        "r"(leader), "h"(static_cast<uint16_t>(3))
        : "memory");
}

}  // namespace gdla
