// Thread-block-cluster helpers for CTA pairs: the CTA's rank, addresses in the peer's
// shared memory, remote mbarrier arrivals, bounded waits on barriers the peer arrives
// on, and one-instruction bulk copies into the peer's shared memory.
#pragma once
#include "tc_utils.cuh"

namespace csa {
namespace cl {

CSA_DEV uint32_t cluster_rank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
CSA_DEV uint32_t peer_addr(uint32_t local_smem_addr, uint32_t peer)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local_smem_addr), "r"(peer));
    return r;
}
CSA_DEV void mbar_arrive_remote(uint32_t remote_bar)
{
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(remote_bar) : "memory");
}
CSA_DEV bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(tc::smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// bounded wait on a barrier that the peer CTA arrives on
CSA_DEV bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, long long budget)
{
    if (mbar_try_wait_cluster(bar, parity)) return true;
    const long long t0 = clock64();
    for (int polls = 0; !mbar_try_wait_cluster(bar, parity); ++polls) {
        if (clock64() - t0 > budget) return false;
        if (polls >= 8) __nanosleep(32);
    }
    return true;
}
// One bulk copy of `bytes` from this CTA's shared memory to a peer CTA's shared memory;
// completion is counted in bytes on the peer's mbarrier.
CSA_DEV void bulk_copy_to_peer(uint32_t dst_cluster, uint32_t src_cta, uint32_t bytes, uint32_t mbar_cluster)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n\t"
        "cp.async.bulk.commit_group;" ::"r"(dst_cluster),
        "r"(src_cta), "r"(bytes), "r"(mbar_cluster)
        : "memory");
}
// Wait until every bulk copy this thread issued has finished reading its source.
CSA_DEV void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
CSA_DEV void cluster_sync()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// ---- CTA pairs on one MMA (cta_group::2): rank 0 of a cluster of two is the leader ----
// TMEM allocation of a CTA pair: both CTAs run it, from the same warp, into the same
// shared memory offset, and receive the same column address.
CSA_DEV void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(tc::smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
CSA_DEV void tmem_relinquish_pair() { asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory"); }
CSA_DEV void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// D (+)= A B^T across the pair, issued by one leader thread: M = 256 rows of A, the
// first 128 from the leader's shared memory and the next 128 from its peer's, both at
// the descriptor's offset; the N rows of B split the same way (N/2 from each CTA).
// Each CTA's TMEM receives its own 128 rows of D for all N columns.
CSA_DEV void mma_bf16_ss_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Once the pair MMAs this thread issued so far complete, arrive once on the barrier at
// bar's offset in every CTA of cta_mask (bit r = cluster rank r).
CSA_DEV void mma_commit_pair(uint64_t* bar, uint16_t cta_mask)
{
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
            tc::smem_u32(bar)),
        "h"(cta_mask)
        : "memory");
}
// 2-D tiled TMA load into this CTA's shared memory whose transaction bytes complete on
// an mbarrier of either CTA of the pair (bar_cluster: a shared::cluster address, e.g.
// the leader's barrier from peer_addr).  No multicast: one destination CTA.
CSA_DEV void tma_load_2d_pair(void* dst, const CUtensorMap* map, uint32_t bar_cluster, int x, int y)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%3, %4}], [%2];" ::"r"(tc::smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(x), "r"(y)
        : "memory");
}

}  // namespace cl
}  // namespace csa
