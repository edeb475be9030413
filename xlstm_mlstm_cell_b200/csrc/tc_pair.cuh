// tc_pair.cuh -- building blocks of kernels that run the 5th-generation tensor cores over a CTA
// pair (tcgen05 with .cta_group::2): the two CTAs of a cluster of two whose ranks differ in bit 0.
//
// One MMA of the pair (issued by one thread of the even-ranked CTA, the leader) computes an
// M = 128 or 256 product whose A rows come half from each CTA (from each CTA's shared memory or
// TMEM at the same offset) and whose B columns come half from each CTA; each CTA receives its half
// of the rows of D, over all N columns, in its own TMEM.  With M = 256 a CTA's 128 rows fill its
// 128 TMEM lanes; with M = 128 a CTA's 64 rows occupy all 128 lanes: lanes 0-63 hold columns
// [0, N/2) and lanes 64-127 hold columns [N/2, N), in N/2 TMEM columns.
#pragma once

#include "tc_common.cuh"

namespace mlstm {
namespace tc {

__device__ __forceinline__ uint32_t cluster_ctarank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_arrive_release() { asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory"); }
__device__ __forceinline__ void cluster_wait_acquire() { asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory"); }

// Shared::cluster address of the object at `local` in the CTA of cluster rank `rank`.
__device__ __forceinline__ uint32_t map_to_rank(const void *local, uint32_t rank)
{
    uint32_t ra;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(smem_u32(local)), "r"(rank));
    return ra;
}

// Arrives on the mbarrier at a shared::cluster address, possibly in the other CTA of the pair.
// The arrivals that cross the pair only hand over shared memory or TMEM that tcgen05 MMAs read or
// write next (the writer fenced it for the async proxy, or for tcgen05, before its CTA's barrier),
// or free it again; the default (CTA-scope) release suffices for that, and the cluster-scope form
// costs the arriving thread a drain of its outstanding memory operations.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar_cluster)
{
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t *bar, uint32_t parity)
{
    return mbar_try_wait(bar, parity);
}

// Bounded wait for a local barrier that the other CTA of the pair arrives on or fills (its
// arrivals, MMA completions and asynchronous stores with byte counts); false once this CTA aborts
// or the limit passes (then the status word is set).
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t *bar, uint32_t parity, const WaitCtx &w)
{
    if (mbar_try_wait_cluster(bar, parity)) return true;
    const unsigned long long t0 = global_timer();
    for (;;) {
        if (mbar_try_wait_cluster(bar, parity)) return true;
        if (*w.abort) return false;
        if (global_timer() - t0 > WAIT_LIMIT_NS) {
            *w.abort = 1u;
            atomicOr(w.status, ERR_TIMEOUT);
            return false;
        }
    }
}

// Bounded wait at cluster scope that ignores the abort flag (teardown).
__device__ __forceinline__ void mbar_wait_cluster_drain(uint64_t *bar, uint32_t parity)
{
    const unsigned long long t0 = global_timer();
    while (!mbar_try_wait_cluster(bar, parity))
        if (global_timer() - t0 > WAIT_LIMIT_NS) return;
}

// 3-D tile load into this CTA's shared memory whose completion (transaction bytes) is counted on
// the mbarrier at a shared::cluster address in either CTA of the pair (no multicast).
__device__ __forceinline__ void tma_load_3d_pair(void *dst, const CUtensorMap *map, int x, int y, int z,
                                                 uint32_t bar_cluster)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];"
        ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar_cluster)
        : "memory");
}

// Stores a float at a shared::cluster address and counts its 4 bytes on the mbarrier at another
// shared::cluster address of the same CTA (asynchronous).
__device__ __forceinline__ void st_async_f32(uint32_t dst_cluster, float v, uint32_t bar_cluster)
{
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];" ::"r"(dst_cluster),
                 "r"(__float_as_uint(v)), "r"(bar_cluster)
                 : "memory");
}

// TMEM allocation over the pair: one warp of each CTA (the same warp index) executes these.
__device__ __forceinline__ void tmem_alloc_pair(uint32_t *dst_smem, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair()
{
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// D[tmem] (+)= A[smem] * B[smem] over the pair (kind::f16: bf16 or fp16 operands).
__device__ __forceinline__ void mma_pair_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem] over the pair with tf32 operands (A: fp32 storage in TMEM).
__device__ __forceinline__ void mma_pair_ts_tf32(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                                 uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::tf32 [%0], [%1], %2, %3, p;\n\t}"
        ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrives once on the mbarrier at a shared::cluster address (this CTA's or the other CTA's of the
// pair) when every MMA issued so far by this thread has completed.
__device__ __forceinline__ void mma_commit_to(uint32_t bar_cluster)
{
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar_cluster)
                 : "memory");
}

}  // namespace tc
}  // namespace mlstm
