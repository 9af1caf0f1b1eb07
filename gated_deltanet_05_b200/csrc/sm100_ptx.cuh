// sm100_ptx.cuh -- thin inline-PTX wrappers for the sm_100a features the prefill kernel
// uses: mbarriers (with bounded waits), TMA tiled loads, tcgen05 MMA / TMEM, and the
// shared-memory matrix descriptors. Written from the public PTX ISA description of
// these instructions. No TMA multicast form is used anywhere.
#pragma once
#include <cuda_fp16.h>
#include <stdint.h>

#include "gdn_common.cuh"

namespace gdn {
namespace sm100 {

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void fence_mbarrier_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Non-blocking probe: has the phase of `bar` with the given parity completed?
__device__ __forceinline__ bool mbar_test(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// The bounded waits below are out of line: they are called from many sites and kept
// out of the instruction cache's way.
// Waits for the phase of `bar` with the given parity to complete. Gives up (returns
// false) after ~limit_cycles SM clocks or as soon as *abort becomes non-zero; on a
// timeout it records kErrTimeout in the device error word and sets *abort.
__device__ __noinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity,
                                                  volatile int *abort, long long limit_cycles)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const long long t0 = clock64();
    while (true) {
        if (mbar_try_wait(bar, parity))
            return true;
        if (*abort)
            return false;
        if (clock64() - t0 > limit_cycles) {
            *abort = 1;
            raise_error(kErrTimeout);
            return false;
        }
    }
}

// Waits for a phase to complete, ignoring any abort request (used to drain async work
// before the CTA exits). Returns false after ~limit_cycles.
__device__ __noinline__ bool mbar_wait_drain(uint64_t *bar, uint32_t parity, long long limit_cycles)
{
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity))
        if (clock64() - t0 > limit_cycles) {
            raise_error(kErrTimeout);
            return false;
        }
    return true;
}

// ---------------------------------------------------------------- fences
__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void named_bar_sync(int id, int n_threads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n_threads) : "memory");
}

// Arrive on a named barrier without waiting (the waiting side uses named_bar_sync with
// the same thread count).
__device__ __forceinline__ void named_bar_arrive(int id, int n_threads)
{
    asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(n_threads) : "memory");
}

// Named barrier that also ANDs a predicate over the participating threads: every
// thread gets the same answer, so a group can take a uniform decision.
__device__ __forceinline__ bool named_bar_and(int id, int n_threads, bool pred)
{
    uint32_t out;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.b32 p, %1, 0;\n\t"
        "bar.red.and.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(out)
        : "r"((uint32_t)pred), "r"(id), "r"(n_threads)
        : "memory");
    return out != 0;
}

// ---------------------------------------------------------------- TMA (no multicast)
__device__ __forceinline__ void tma_prefetch_desc(const void *desc)
{
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(desc)) : "memory");
}

// 3-D tiled load of one box into shared memory; completion is signalled as transaction
// bytes on `bar`. Coordinates are element indices, innermost first.
__device__ __forceinline__ void tma_load_3d(void *smem_dst, const void *desc, uint64_t *bar, int c0,
                                            int c1, int c2)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(desc)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}

// 3-D tiled store of one box from shared memory, tracked by this thread's bulk
// async-group. Coordinates are element indices, innermost first, all >= 0; rows of the
// box beyond the tensor's extent are not written.
__device__ __forceinline__ void tma_store_3d(const void *desc, const void *smem_src, int c0, int c1, int c2)
{
    asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(desc)),
                 "r"(smem_u32(smem_src)), "r"(c0), "r"(c1), "r"(c2)
                 : "memory");
}

// Bulk (non-tensor) copy shared -> global, tracked by this thread's bulk async-group.
// Both addresses 16-byte aligned, size a multiple of 16.
__device__ __forceinline__ void bulk_store_s2g(void *gdst, const void *ssrc, uint32_t bytes)
{
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst),
                 "r"(smem_u32(ssrc)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// All of this thread's bulk copies have finished reading shared memory.
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// All of this thread's bulk copies have completed.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// ---------------------------------------------------------------- thread-block clusters
__device__ __forceinline__ uint32_t cluster_ctarank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Shared-memory address of the same offset in CTA `rank` of this cluster.
__device__ __forceinline__ uint32_t map_to_peer(uint32_t local_smem_addr, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local_smem_addr), "r"(rank));
    return r;
}

// Arrive (release at cluster scope) on an mbarrier of another CTA of the cluster.
__device__ __forceinline__ void mbar_arrive_remote(uint32_t remote_bar)
{
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(remote_bar) : "memory");
}
// Relaxed variant: for signals that publish no memory writes of the arriving thread (so
// it does not wait for the thread's outstanding stores).
__device__ __forceinline__ void mbar_arrive_remote_relaxed(uint32_t remote_bar)
{
    asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(remote_bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx_remote_relaxed(uint32_t remote_bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.relaxed.cluster.shared::cluster.b64 _, [%0], %1;" ::"r"(remote_bar),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx_remote(uint32_t remote_bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.release.cluster.shared::cluster.b64 _, [%0], %1;" ::"r"(remote_bar),
                 "r"(bytes)
                 : "memory");
}

// Waits, with cluster-scope acquire, for a phase of a local mbarrier that another CTA of
// the cluster signals. Bounded like mbar_wait_bounded.
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ bool mbar_test_cluster(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __noinline__ bool mbar_wait_cluster_bounded(uint64_t *bar, uint32_t parity, volatile int *abort,
                                                          long long limit_cycles)
{
    const long long t0 = clock64();
    while (!mbar_try_wait_cluster(bar, parity)) {
        if (*abort) return false;
        if (clock64() - t0 > limit_cycles) {
            *abort = 1;
            raise_error(kErrTimeout);
            return false;
        }
    }
    return true;
}

// The slow path of a kernel role's wait, out of line so that each call site stays a probe
// and a call: a bounded wait with acquire at cluster scope (cluster != 0) or CTA scope; when
// it gives up (a timeout, or the abort flag already raised) it also raises the other CTA's
// abort flag (peer_abort, a shared::cluster address) so that both CTAs of the cluster stop.
__device__ __noinline__ bool mbar_wait_or_abort(uint64_t *bar, uint32_t parity, volatile int *abort,
                                                uint32_t peer_abort, uint32_t cluster, long long limit_cycles)
{
    const bool ok = cluster ? mbar_wait_cluster_bounded(bar, parity, abort, limit_cycles)
                            : mbar_wait_bounded(bar, parity, abort, limit_cycles);
    if (!ok) asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(peer_abort), "r"(1u) : "memory");
    return ok;
}

// Bulk copy from this CTA's shared memory into another CTA's shared memory of the
// cluster; completion is counted as transaction bytes on the destination's mbarrier.
// No multicast. Addresses 16-byte aligned, size a multiple of 16.
__device__ __forceinline__ void bulk_copy_s2peer(uint32_t remote_dst, const void *local_src, uint32_t bytes,
                                                 uint32_t remote_bar)
{
    asm volatile("cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
                     "r"(remote_dst),
                 "r"(smem_u32(local_src)), "r"(bytes), "r"(remote_bar)
                 : "memory");
}
// 32-bit load from another CTA's shared memory (address from map_to_peer).
__device__ __forceinline__ uint32_t ld_cluster_u32(uint32_t remote_addr)
{
    uint32_t v;
    asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(remote_addr) : "memory");
    return v;
}

// Bulk copy global -> this CTA's shared memory, completing as transaction bytes on `bar`.
// Addresses 16-byte aligned, size a multiple of 16.
__device__ __forceinline__ void bulk_load_g2s(void *sdst, const void *gsrc, uint32_t bytes, uint64_t *bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(sdst)),
                 "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}
// Bulk copies of this thread: at most one group not yet complete.
__device__ __forceinline__ void bulk_wait_all_but_1() { asm volatile("cp.async.bulk.wait_group 1;" ::: "memory"); }
// Orders this thread's generic-proxy view of global memory with async-proxy (bulk/TMA)
// accesses.
__device__ __forceinline__ void fence_proxy_async_global()
{
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

__device__ __forceinline__ uint32_t smid()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(r));
    return r;
}

__device__ __forceinline__ bool elect_one()
{
    uint32_t p;
    asm volatile("{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\tselp.b32 %0, 1, 0, e;\n\t}" : "=r"(p));
    return p != 0;
}

// 32-bit store into another CTA's shared memory (address from map_to_peer).
__device__ __forceinline__ void st_cluster_u32(uint32_t remote_addr, uint32_t v)
{
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(remote_addr), "r"(v) : "memory");
}

__device__ __forceinline__ void cluster_sync_all()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// ---------------------------------------------------------------- tcgen05 / TMEM
__device__ __forceinline__ void tmem_alloc(uint32_t *smem_slot, uint32_t n_cols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(smem_slot)),
                 "r"(n_cols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish()
{
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t n_cols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(n_cols)
                 : "memory");
}

// D[tmem] (+)= A[smem desc] x B[smem desc], kind::f16 (f16 or bf16 inputs per the
// instruction descriptor, fp32 accumulate).
__device__ __forceinline__ void mma_f16kind_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// D[tmem] (+)= A[tmem] x B[smem desc], kind::f16. A is M x K with row m in TMEM lane m and
// two 16-bit K elements per 32-bit column (lower K index in the low half); a K step of 16
// advances the A address by 8 columns. A is K-major by construction (descriptor bit 15 = 0).
__device__ __forceinline__ void mma_f16kind_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Leader-predicated forms: executed by a whole converged warp with warp-uniform operands
// (so they stay in uniform registers); only the lane with `leader` != 0 issues. Keeping the
// warp converged avoids per-lane operand loops around these instructions.
__device__ __forceinline__ void mma_ss_lead(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate, uint32_t leader)
{
    asm volatile(
        "{\n\t.reg .pred p, l;\n\t"
        "setp.ne.b32 p, %4, 0;\n\tsetp.ne.b32 l, %5, 0;\n\t"
        "@l tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(leader)
        : "memory");
}
__device__ __forceinline__ void mma_ts_lead(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate, uint32_t leader)
{
    asm volatile(
        "{\n\t.reg .pred p, l;\n\t"
        "setp.ne.b32 p, %4, 0;\n\tsetp.ne.b32 l, %5, 0;\n\t"
        "@l tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(leader)
        : "memory");
}
__device__ __forceinline__ void mma_commit_lead(uint64_t *bar, uint32_t leader)
{
    asm volatile(
        "{\n\t.reg .pred l;\n\tsetp.ne.b32 l, %1, 0;\n\t"
        "@l tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(smem_u32(bar)),
        "r"(leader)
        : "memory");
}
__device__ __forceinline__ void tma_load_3d_lead(void *smem_dst, const void *desc, uint64_t *bar, int c0, int c1,
                                                 int c2, uint32_t leader)
{
    asm volatile(
        "{\n\t.reg .pred l;\n\tsetp.ne.b32 l, %6, 0;\n\t"
        "@l cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];\n\t}" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(desc)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(leader)
        : "memory");
}
__device__ __forceinline__ void tma_load_2d_lead(void *smem_dst, const void *desc, uint64_t *bar, int c0, int c1,
                                                 uint32_t leader)
{
    asm volatile(
        "{\n\t.reg .pred l;\n\tsetp.ne.b32 l, %5, 0;\n\t"
        "@l cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];\n\t}" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(desc)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(leader)
        : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx_lead(uint64_t *bar, uint32_t bytes, uint32_t leader)
{
    asm volatile(
        "{\n\t.reg .pred l;\n\tsetp.ne.b32 l, %2, 0;\n\t"
        "@l mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n\t}" ::"r"(smem_u32(bar)),
        "r"(bytes), "r"(leader)
        : "memory");
}
__device__ __forceinline__ void bulk_load_g2s_lead(void *sdst, const void *gsrc, uint32_t bytes, uint64_t *bar,
                                                   uint32_t leader)
{
    asm volatile(
        "{\n\t.reg .pred l;\n\tsetp.ne.b32 l, %4, 0;\n\t"
        "@l cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n\t}" ::"r"(
            smem_u32(sdst)),
        "l"(gsrc), "r"(bytes), "r"(smem_u32(bar)), "r"(leader)
        : "memory");
}
__device__ __forceinline__ void mbar_arrive_lead(uint64_t *bar, uint32_t leader)
{
    asm volatile(
        "{\n\t.reg .pred l;\n\tsetp.ne.b32 l, %1, 0;\n\t"
        "@l mbarrier.arrive.shared::cta.b64 _, [%0];\n\t}" ::"r"(smem_u32(bar)),
        "r"(leader)
        : "memory");
}
__device__ __forceinline__ void mbar_arrive_remote_lead(uint32_t remote_bar, uint32_t leader)
{
    asm volatile(
        "{\n\t.reg .pred l;\n\tsetp.ne.b32 l, %1, 0;\n\t"
        "@l mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];\n\t}" ::"r"(remote_bar),
        "r"(leader)
        : "memory");
}
__device__ __forceinline__ void bulk_store_s2g_lead(void *gdst, const void *ssrc, uint32_t bytes, uint32_t leader)
{
    asm volatile(
        "{\n\t.reg .pred l;\n\tsetp.ne.b32 l, %3, 0;\n\t"
        "@l cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;\n\t}" ::"l"(gdst),
        "r"(smem_u32(ssrc)), "r"(bytes), "r"(leader)
        : "memory");
}
__device__ __forceinline__ void mbar_arrive_remote_relaxed_lead(uint32_t remote_bar, uint32_t leader)
{
    asm volatile(
        "{\n\t.reg .pred l;\n\tsetp.ne.b32 l, %1, 0;\n\t"
        "@l mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];\n\t}" ::"r"(remote_bar),
        "r"(leader)
        : "memory");
}

// Arrive once on `bar` when every tcgen05 operation this thread issued so far is done.
__device__ __forceinline__ void mma_commit(uint64_t *bar)
{
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld_x32(uint32_t taddr, uint32_t (&r)[32])
{
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
                 : "r"(taddr));
}

__device__ __forceinline__ void tmem_st_x32(uint32_t taddr, const uint32_t (&r)[32])
{
    asm volatile("tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
                 :: "r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
                 : "memory");
}

__device__ __forceinline__ void tmem_ld_x8(uint32_t taddr, uint32_t (&r)[8])
{
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld_x16(uint32_t taddr, uint32_t (&r)[16])
{
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
                 : "r"(taddr));
}

__device__ __forceinline__ void tmem_st_x16(uint32_t taddr, const uint32_t (&r)[16])
{
    asm volatile("tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
                 :: "r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
                 : "memory");
}

// Instruction descriptor of tcgen05.mma kind::f16 with fp32 D. A and B share one input
// type: `ab_format` 0 = f16, 1 = bf16.
// Bits: [4,6) D format (1 = f32); [7,10) A format; [10,13) B format; 15 A major (0 = K,
// 1 = MN); 16 B major; [17,23) N >> 3; [24,29) M >> 4.
__host__ __device__ constexpr uint32_t idesc_f32acc(int ab_format, int M, int N, int a_mn_major,
                                                    int b_mn_major)
{
    return (1u << 4) | ((uint32_t)ab_format << 7) | ((uint32_t)ab_format << 10) |
           ((uint32_t)a_mn_major << 15) | ((uint32_t)b_mn_major << 16) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}
constexpr int kFmtF16 = 0, kFmtBF16 = 1;

// Shared-memory matrix descriptor for a 128-byte-swizzled operand tile.
// Bits: [0,14) start address >> 4; [16,30) leading byte offset >> 4; [32,46) stride
// byte offset >> 4; [46,48) descriptor version (1); [49,52) base offset (0: tiles are
// 1024-byte aligned); [61,64) layout (2 = 128-byte swizzle).
// K-major tiles: rows of 128 bytes (64 bf16 along K), 8-row groups SBO bytes apart;
// MN-major tiles: rows of 128 bytes (64 bf16 along M or N) indexed by K, 8-row groups
// SBO bytes apart, 64-element M/N blocks LBO bytes apart.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t smem_addr, uint32_t lbo_bytes,
                                                uint32_t sbo_bytes)
{
    uint64_t d = 0;
    d |= (uint64_t)((smem_addr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

// Byte offset of 16-byte chunk `c` (0..7) of row `r` inside a 128-byte-swizzled tile.
__device__ __forceinline__ uint32_t sw128_off(int r, int c) { return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4)); }

// ---------------------------------------------------------------- warp-level MMA
// D = A x B + D for one 16x8x8 tile, tf32 inputs, fp32 accumulate (mma.sync). Used for
// the small block products of the triangular solve, where the M >= 64 of tcgen05 does
// not fit. Fragment ownership (g = lane / 4, q = lane % 4):
//   A 16x8 row-major: a0 (g, q), a1 (g+8, q), a2 (g, q+4), a3 (g+8, q+4)
//   B 8x8 (k x n):    b0 (q, g), b1 (q+4, g)
//   D 16x8:           d0 (g, 2q), d1 (g, 2q+1), d2 (g+8, 2q), d3 (g+8, 2q+1)
__device__ __forceinline__ void mma_tf32_16x8x8(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2])
{
    asm volatile("mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                 "{%0,%1,%2,%3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

__device__ __forceinline__ uint32_t to_tf32(float x)
{
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}

// 2^x with the SM's approximate base-2 exponential instruction (denormal results flush
// to zero). Every argument here is <= 0, so results lie in [0, 1].
__device__ __forceinline__ float fast_exp2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi)
{
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

// fp16 range checks. The tensor-core products take fp16 operands, which hold |x| < 65520
// (larger values round to inf). f16x2_absmax keeps, per 16-bit half, the largest magnitude
// bit pattern seen (sign cleared); a finite fp16 has a pattern below 0x7c00, inf and NaN do
// not, so f16x2_overflowed tells whether any packed value converted so far overflowed.
__device__ __forceinline__ uint32_t f16x2_absmax(uint32_t acc, uint32_t w) { return __vmaxu2(acc, w & 0x7fff7fffu); }
__device__ __forceinline__ uint32_t f16x8_absmax(uint32_t acc, uint4 w)
{
    return f16x2_absmax(f16x2_absmax(acc, w.x), __vmaxu2(w.y & 0x7fff7fffu, __vmaxu2(w.z & 0x7fff7fffu, w.w & 0x7fff7fffu)));
}
__device__ __forceinline__ bool f16x2_overflowed(uint32_t acc)
{
    return (acc & 0xffffu) >= 0x7c00u || (acc >> 16) >= 0x7c00u;
}
// max(acc, |x|) that propagates NaN (so a NaN also fails the final range test).
__device__ __forceinline__ float max_abs_nan(float acc, float x)
{
    float r;
    asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(acc), "f"(fabsf(x)));
    return r;
}
constexpr float kF16Limit = 65520.f;   // fp16 round-to-nearest overflows at and above this

}  // namespace sm100
}  // namespace gdn
