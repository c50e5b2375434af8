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

}  // namespace cl
}  // namespace csa
