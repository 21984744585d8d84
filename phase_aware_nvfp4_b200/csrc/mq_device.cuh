// mq_device.cuh -- sm_100a device helpers: mbarriers with bounded waits, TMA and
// bulk copies, tcgen05 (TMEM alloc, UMMA, SMEM->TMEM copy, TMEM loads), and
// the NVFP4 number-format helpers the kernels share.
//
// Everything here is written against the public PTX ISA for sm_100a.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <utility>

#include "mq_internal.h"

namespace mq {

// --------------------------------------------------------------------------
// Generic
// --------------------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void* p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Post an asynchronous error bit to the workspace control block.
__device__ __forceinline__ void post_error(WsControl* ctrl, uint32_t bit)
{
    if (ctrl != nullptr) atomicOr(&ctrl->error_bits, bit);
}

// --------------------------------------------------------------------------
// mbarrier
// --------------------------------------------------------------------------

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbarrier_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar_addr, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar_addr), "r"(parity)
        : "memory");
    return ok != 0;
}

// try_wait with a suspend-time hint: a thread whose phase is not complete
// sleeps until it completes (or the hint expires) instead of spinning.
__device__ __forceinline__ bool mbar_try_wait_hint(uint32_t bar_addr, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar_addr), "r"(parity), "r"(0x989680u)
        : "memory");
    return ok != 0;
}

// Non-blocking test of a phase: never suspends the thread.  Used to look at
// the next pipeline stage before issuing the current stage's tensor-core work,
// so the barrier's shared-memory round trip overlaps that work.
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity)
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

// Wait until the phase with the given parity has completed.  Bounded: gives
// up after kWaitTimeoutNs of wall time and returns false, so a lost arrival
// turns into an error status instead of a hung GPU.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint64_t timeout_ns = kWaitTimeoutNs)
{
    const uint32_t a = smem_u32(bar);
    if (mbar_try_wait_hint(a, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        if (mbar_try_wait_hint(a, parity)) return true;
        if (globaltimer_ns() - t0 > timeout_ns) return false;
    }
}

// Warp-uniform forms, for loops that a whole converged warp runs so that its
// values stay warp-uniform (the tensor-core instructions issued from such a
// loop under elect_one() read their operands from uniform registers).
// Every lane observes the phase itself; the vote makes the result (and so
// the control flow after it) identical across the warp.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile uint32_t* abort_flag,
                                          uint64_t timeout_ns = kWaitTimeoutNs)
{
    const bool ok = !*abort_flag && mbar_wait(bar, parity, timeout_ns);
    return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ bool warp_test(uint64_t* bar, uint32_t parity)
{
    return __all_sync(0xffffffffu, mbar_test_wait(bar, parity));
}

// One lane of the converged warp is elected (elect.sync).
__device__ __forceinline__ bool elect_one()
{
    uint32_t pred;
    asm volatile(
        "{\n\t.reg .pred P;\n\t"
        "elect.sync _|P, 0xffffffff;\n\t"
        "selp.u32 %0, 1, 0, P;\n\t}"
        : "=r"(pred));
    return pred != 0;
}

// Programmatic dependent launch (sm_90+).  A kernel launched with
// programmatic stream serialization may start before the previous kernel in
// the stream has finished; grid_dep_wait() blocks the calling thread until
// that kernel has completed and its memory operations are visible, and
// grid_dep_launch_dependents() lets the next kernel start early.  Both are
// no-ops when the launch has no such dependency.
// Ticket of a "last one folds" hand-off between CTAs: an atomic add with
// acquire-release semantics at GPU scope.  The release orders the caller's
// earlier writes, and (being cumulative) those its CTA made before a barrier
// with the caller, before the increment; the acquire makes every write that
// the earlier incrementers released visible after it, to the caller and to its
// CTA after a barrier.  No full fence is needed around it.
__device__ __forceinline__ uint32_t atom_add_acq_rel_gpu(uint32_t* p, uint32_t v)
{
    uint32_t old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}

// Relaxed (not ordering) read of a 32-bit word written by other CTAs.
__device__ __forceinline__ uint32_t ld_relaxed_gpu_u32(const uint32_t* p)
{
    uint32_t v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;"); }

// Host side: launch `kern` with programmatic stream serialization, so its
// CTAs may be scheduled (and run their set-up) while the previous kernel in
// the stream drains.  Every kernel launched this way calls grid_dep_wait()
// before its first access to global memory that another kernel may write,
// so the stream order of memory effects is unchanged.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args&&... args)
{
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
    return e != cudaSuccess ? e : cudaGetLastError();
}

// --------------------------------------------------------------------------
// TMA / bulk copies (global -> shared, completion on an mbarrier)
// --------------------------------------------------------------------------

__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map, uint64_t* bar, int32_t x,
                                            int32_t y)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::
            "r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
        : "memory");
}

// Prefetch `bytes` (a multiple of 16, 16-byte aligned source) into L2.
__device__ __forceinline__ void bulk_prefetch_l2(const void* gsrc, uint32_t bytes)
{
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(gsrc), "r"(bytes) : "memory");
}

__device__ __forceinline__ void bulk_load(void* smem_dst, const void* gsrc, uint32_t bytes, uint64_t* bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(smem_dst)),
                 "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

// TMA tile store shared -> global (bulk-group completion), and its fences.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* smem_src, int32_t x, int32_t y)
{
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(smem_u32(smem_src)), "r"(x), "r"(y)
                 : "memory");
}

__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

// Wait until at most N committed bulk groups still read their shared-memory source.
template <int N>
__device__ __forceinline__ void bulk_wait_group_read()
{
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

// Wait until at most N committed bulk groups are still in flight.
template <int N>
__device__ __forceinline__ void bulk_wait_group()
{
    asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}

// Make this thread's generic-proxy shared-memory writes visible to the async proxy (TMA).
__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void named_barrier_sync(uint32_t id, uint32_t nthreads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map)
{
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// --------------------------------------------------------------------------
// tcgen05
// --------------------------------------------------------------------------

// Allocate `ncols` TMEM columns (power of two >= 32); the base address is
// written to shared memory.  Executed by one whole warp.
__device__ __forceinline__ void tmem_alloc(uint32_t* smem_dst, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(smem_dst)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before()
{
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after()
{
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Arrive on `bar` once every tcgen05 operation issued so far by this thread
// has completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// Block-scaled FP4 x FP4 -> FP32 UMMA, 16-element scale blocks (NVFP4).
__device__ __forceinline__ void umma_nvfp4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                           uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
            d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
}

// BF16 x BF16 -> FP32 UMMA.
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Copy a 32-row x 16-byte block from shared memory into TMEM lanes 0..31 of
// 4 consecutive columns, replicated into all four 32-lane sub-partitions.
__device__ __forceinline__ void tmem_cp_32x128b_x4(uint32_t taddr, uint64_t sdesc)
{
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

__device__ __forceinline__ void tmem_wait_ld()
{
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Wait for the TMEM loads, then pass the destination registers through empty
// volatile asm statements: their later uses depend on those, so the compiler
// cannot move a use of a loaded register above the wait.
template <int N>
__device__ __forceinline__ void tmem_wait_ld(uint32_t (&r)[N])
{
    tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < N; ++i) asm volatile("" : "+r"(r[i]));
}

// Each thread of the warp reads 32 consecutive 32-bit columns of its own
// TMEM lane (lane = 32 * (warp % 4) + laneid, encoded in taddr[31:16]).
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]),
          "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
          "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}

// Each thread reads 16 consecutive 32-bit columns of its TMEM lane.
__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

// --------------------------------------------------------------------------
// CTA pairs (tcgen05 cta_group::2): one MMA spans the tensor cores of two SMs
// --------------------------------------------------------------------------

__device__ __forceinline__ uint32_t cluster_ctarank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_barrier()
{
    asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}

// Shared::cluster address of the same shared-memory offset in CTA `rank`.
__device__ __forceinline__ uint32_t map_to_cta(uint32_t smem_addr, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr), "r"(rank));
    return r;
}

// Arrive on an mbarrier that may live in another CTA of the cluster.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr)
{
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// Store a 32-bit value into shared memory of a CTA of the cluster
// (cluster_addr from map_to_cta).
__device__ __forceinline__ void st_cluster_u32(uint32_t cluster_addr, uint32_t v)
{
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(cluster_addr), "r"(v) : "memory");
}

// Bounded wait on a local mbarrier whose arrivals come from other CTAs of the
// cluster (acquire at cluster scope, so their stores before a release arrive
// are visible afterwards).
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity,
                                                  uint64_t timeout_ns = kWaitTimeoutNs)
{
    const uint32_t a = smem_u32(bar);
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        uint32_t ok;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok)
            : "r"(a), "r"(parity)
            : "memory");
        if (ok) return true;
        if (globaltimer_ns() - t0 > timeout_ns) return false;
    }
}

// TMA tile load into this CTA's shared memory whose completion is signalled
// on an mbarrier of either CTA of the pair (bar = shared::cluster address).
__device__ __forceinline__ void tma_load_2d_pair(void* smem_dst, const CUtensorMap* map, uint32_t bar, int32_t x,
                                                 int32_t y)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
        "%4}], [%2];" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y)
        : "memory");
}

// 3-D form of the pair load (x innermost).
__device__ __forceinline__ void tma_load_3d_pair(void* smem_dst, const CUtensorMap* map, uint32_t bar, int32_t x,
                                                 int32_t y, int32_t z)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
        "%4, %5}], [%2];" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y), "r"(z)
        : "memory");
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t* smem_dst, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(smem_dst)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// Block-scaled NVFP4 UMMA over the CTA pair: M = 256 (128 rows of A from each
// CTA), B rows split between the two CTAs, D and scale factors in each CTA's TMEM.
__device__ __forceinline__ void umma_nvfp4_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                                uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
            d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
}

// 32 x 128-bit SMEM -> TMEM copy performed in both CTAs of the pair (each
// CTA's shared memory into its own TMEM, same addresses).
__device__ __forceinline__ void tmem_cp_32x128b_x4_pair(uint32_t taddr, uint64_t sdesc)
{
    asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// Arrive on the mbarrier at the same offset in every CTA of `cta_mask` once
// all pair-MMAs / copies issued so far by this thread have completed.
__device__ __forceinline__ void tc_commit_pair_mc(uint64_t* bar, uint16_t cta_mask)
{
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
                     smem_u32(bar)),
                 "h"(cta_mask)
                 : "memory");
}

__device__ __forceinline__ void tc_commit_pair(uint64_t* bar)
{
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

// --------------------------------------------------------------------------
// UMMA descriptors
// --------------------------------------------------------------------------

// Shared-memory matrix descriptor, K-major operand with the 128-byte swizzle
// (rows of 128 bytes, 8-row atoms of 1024 bytes).  Fields: start address
// >> 4 in [0,14), leading byte offset >> 4 in [16,30) (unused for this
// layout, 1), stride byte offset >> 4 in [32,46) (1024 bytes between 8-row
// groups), descriptor version 1 in [46,48), swizzle mode 2 (128B) in [61,64).
__device__ __forceinline__ uint64_t sdesc_kmajor_sw128(uint32_t saddr)
{
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1u << 16) | ((uint64_t)(1024u >> 4) << 32) |
           ((uint64_t)1u << 46) | ((uint64_t)2u << 61);
}

// Descriptor of a plain (unswizzled) 32-row x 16-byte block for tcgen05.cp:
// 8-row core matrices of 128 contiguous bytes, 128 bytes apart.
__device__ __forceinline__ uint64_t sdesc_sf_block(uint32_t saddr)
{
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)(128u >> 4) << 32) | ((uint64_t)1u << 46);
}

// Instruction descriptor for kind::mxf4nvf4: A and B E2M1 (format 1), K-major,
// UE4M3 scales (format 0), dense, MMA_K = 64; N >> 3 in [17,23), M >> 4 in
// [24,29).
__host__ __device__ constexpr uint32_t idesc_nvfp4(int M, int N)
{
    return (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Instruction descriptor for kind::f16 with BF16 A/B (format 1), FP32 D
// (format 1 in [4,6)), K-major A and B.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N)
{
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// --------------------------------------------------------------------------
// Number formats (NVFP4 quantizer arithmetic on the device)
// --------------------------------------------------------------------------

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Round a non-negative FP32 block scale onto the E4M3 grid: nearest, ties
// to even, saturating at 448 (the PTX cvt with .satfinite does exactly that
// for finite inputs; the clamp keeps +inf out of it).
__device__ __forceinline__ uint32_t e4m3_round_sat(float s)
{
    s = fminf(s, 448.0f);
    uint16_t pair;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(pair) : "f"(0.0f), "f"(s));
    return (uint32_t)(pair & 0xFFu);
}

// Value of a non-negative E4M3 code (never NaN here: codes <= 0x7E).
__device__ __forceinline__ float e4m3_to_float(uint32_t c)
{
    const uint32_t e = (c >> 3) & 15u, m = c & 7u;
    if (e == 0u) return (float)m * 0.001953125f;  // m * 2^-9, exact
    return __uint_as_float(((e + 120u) << 23) | (m << 20));
}

// Index 0..7 of the E2M1 magnitude nearest to m >= 0 (ties to even index,
// clipped at 6): count the decision thresholds m lies above.  A threshold
// that sits between an even and an odd index sends its tie to the even one.
__device__ __forceinline__ uint32_t e2m1_index(float m)
{
    return (uint32_t)(m > 0.25f) + (uint32_t)(m >= 0.75f) + (uint32_t)(m > 1.25f) + (uint32_t)(m >= 1.75f) +
           (uint32_t)(m > 2.5f) + (uint32_t)(m >= 3.5f) + (uint32_t)(m > 5.0f);
}

// 4-bit code of one element: sign bit of x, magnitude index of |x| * enc.
// (Definition-based form; the kernels use the conversion instruction below,
// and the self-test checks the two agree on every input.)
__device__ __forceinline__ uint32_t e2m1_code(float x, float enc)
{
    const float a = fabsf(x);
    const uint32_t idx = (a == 0.0f) ? 0u : e2m1_index(__fmul_rn(a, enc));
    return ((__float_as_uint(x) >> 28) & 8u) | idx;
}

// Eight E2M1 codes packed into 32 bits (element j in bits 4j..4j+3) from
// eight already-scaled values, by the sm_100 conversion instruction: round
// to nearest even on the E2M1 grid, saturating at +-6, sign kept (also on
// zero).  Each cvt packs two values: the first source lands in the upper
// nibble.
__device__ __forceinline__ uint32_t e2m1x8_cvt(float v0, float v1, float v2, float v3, float v4, float v5,
                                               float v6, float v7)
{
    uint32_t out;
    asm("{\n\t.reg .b8 q0, q1, q2, q3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q3, %8, %7;\n\t"
        "mov.b32 %0, {q0, q1, q2, q3};\n\t}"
        : "=r"(out)
        : "f"(v0), "f"(v1), "f"(v2), "f"(v3), "f"(v4), "f"(v5), "f"(v6), "f"(v7));
    return out;
}

// Two binary32 products in one instruction (mul.rn.f32x2, sm_100): each lane
// is the correctly rounded product, as __fmul_rn (no flush of subnormals).
__device__ __forceinline__ void fmul2_rn(float a0, float a1, float b, float& d0, float& d1)
{
    uint64_t d;
    const uint64_t a = ((uint64_t)__float_as_uint(a1) << 32) | __float_as_uint(a0);
    const uint64_t bb = ((uint64_t)__float_as_uint(b) << 32) | __float_as_uint(b);
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(bb));
    d0 = __uint_as_float((uint32_t)d);
    d1 = __uint_as_float((uint32_t)(d >> 32));
}

// Two binary32 products of two pairs, (a0 * b0, a1 * b1), in one instruction.
__device__ __forceinline__ void fmul2v_rn(float a0, float a1, float b0, float b1, float& d0, float& d1)
{
    uint64_t d;
    const uint64_t a = ((uint64_t)__float_as_uint(a1) << 32) | __float_as_uint(a0);
    const uint64_t b = ((uint64_t)__float_as_uint(b1) << 32) | __float_as_uint(b0);
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    d0 = __uint_as_float((uint32_t)d);
    d1 = __uint_as_float((uint32_t)(d >> 32));
}

// Codes of eight values x[0..7] with encode scale enc = fl(1 / fl(alpha * sigma)):
// code = Pi_FP4(x * enc) with the sign of x.  When enc overflowed to +inf
// (alpha * sigma below 2^-128) a zero x would give 0 * inf = NaN, so that rare
// block takes the element-wise path, which maps zeros to a signed zero code.
__device__ __forceinline__ uint32_t e2m1x8_encode(const float (&x)[8], float enc)
{
    if (isinf(enc)) {
        uint32_t out = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) out |= e2m1_code(x[j], enc) << (4 * j);
        return out;
    }
    float m[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) fmul2_rn(x[2 * j], x[2 * j + 1], enc, m[2 * j], m[2 * j + 1]);
    return e2m1x8_cvt(m[0], m[1], m[2], m[3], m[4], m[5], m[6], m[7]);
}

// Per-halfword unsigned maximum (PTX max.u16x2).  The magnitude bits of a
// non-negative bf16 order like the values, so this is a two-wide |bf16| max.
__device__ __forceinline__ uint32_t max_u16x2(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// Per-lane max(|a|, |b|) of two BF16 pairs (max.xorsign.abs.bf16x2): the
// magnitude is exact; the sign bit (xor of the inputs' signs) is discarded by
// the caller.
__device__ __forceinline__ uint32_t max_abs_bf16x2(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// |bf16| maximum of 16 values held as 8 packed words (exact for finite values;
// a non-finite input is reported by the amax pass and its block is not
// required to match anything).
__device__ __forceinline__ float bf16x16_absmax(const uint32_t (&w)[8])
{
    const uint32_t m = max_abs_bf16x2(max_abs_bf16x2(max_abs_bf16x2(w[0], w[1]), max_abs_bf16x2(w[2], w[3])),
                                      max_abs_bf16x2(max_abs_bf16x2(w[4], w[5]), max_abs_bf16x2(w[6], w[7])));
    const uint32_t b = max(m & 0x7FFFu, (m >> 16) & 0x7FFFu);
    return __uint_as_float(b << 16);
}

// Per-halfword |bf16| maximum over the finite values of a 32-bit word pair,
// plus a flag word that is non-zero if a NaN/Inf was seen.
__device__ __forceinline__ void amax_accum(uint32_t w, uint32_t& mx, uint32_t& bad)
{
    const uint32_t mag = w & 0x7FFF7FFFu;
    const uint32_t nonfin = __vcmpgeu2(mag, 0x7F807F80u);  // 0xFFFF per NaN/Inf halfword
    bad |= nonfin;
    mx = max_u16x2(mx, mag & ~nonfin);
}

// Fold of two (|bf16| maximum, non-finite flag in bit 31) words.
__device__ __forceinline__ uint32_t fold_max_flag(uint32_t a, uint32_t b)
{
    return max(a & 0x7FFFFFFFu, b & 0x7FFFFFFFu) | ((a | b) & 0x80000000u);
}

// E4M3 codes (RNE, satfinite) of two non-negative values in one conversion:
// low byte = code of lo, next byte = code of hi.
__device__ __forceinline__ uint32_t e4m3x2_round_sat(float lo, float hi)
{
    uint16_t pair;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(pair) : "f"(fminf(hi, 448.0f)), "f"(fminf(lo, 448.0f)));
    return pair;
}

// Eq. 3 block scale code Pi_E4M3(fl(amax / aq)) without a division on the
// common path.  inv_lo <= 1/aq <= inv_hi are adjacent floats, so the exact
// quotient lies in [amax*inv_lo, amax*inv_hi]; rounding is monotone, hence
// fl(amax/aq) lies between the two rounded products and, when both round to
// the same E4M3 code, so does it.  Otherwise (a product pair straddling an
// E4M3 rounding boundary) the correctly rounded division decides.
__device__ __forceinline__ uint32_t e4m3_block_scale(float amax, float aq, float inv_lo, float inv_hi)
{
    const uint32_t pair = e4m3x2_round_sat(__fmul_rn(amax, inv_lo), __fmul_rn(amax, inv_hi));
    const uint32_t c = pair & 0xFFu;
    if (c == (pair >> 8)) return c;
    return e4m3_round_sat(__fdiv_rn(amax, aq));
}

// Per-block constants of the Eq. 2 / Eq. 3 arithmetic for one tensor scale.
struct QuantConsts {
    float alpha_qmax;       // fl(alpha * q_max)
    float inv_lo, inv_hi;   // floats bracketing 1 / alpha_qmax (see e4m3_block_scale)
};

__device__ __forceinline__ QuantConsts quant_consts(float alpha)
{
    QuantConsts q;
    q.alpha_qmax = __fmul_rn(alpha, 6.0f);
    // When fl(1/alpha_qmax) is not a normal finite float the bracket [0, inf]
    // sends every block to the exact division.
    const float inv_near = __frcp_rn(q.alpha_qmax);
    const bool inv_normal = inv_near >= 1.17549435e-38f && inv_near < 3.0e38f;
    q.inv_lo = inv_normal ? __uint_as_float(__float_as_uint(inv_near) - 1u) : 0.0f;
    q.inv_hi = inv_normal ? __uint_as_float(__float_as_uint(inv_near) + 1u) : __int_as_float(0x7F800000);
    return q;
}

// Eq. 3 scale code and Eq. 2 codes of one 16-element block held as eight BF16
// pairs (element 2j in the low half of w[j]); enc_tab[c] = fl(1 / fl(alpha * sigma_c)).
// Codes: element j of the block in nibble j of c0 (j < 8) or c1 (j - 8).
__device__ __forceinline__ uint32_t quant_block16(const uint32_t (&w)[8], const QuantConsts& qc,
                                                  const float* enc_tab, uint32_t& c0, uint32_t& c1)
{
    const float amax = bf16x16_absmax(w);
    const uint32_t sc = e4m3_block_scale(amax, qc.alpha_qmax, qc.inv_lo, qc.inv_hi);
    const float enc = enc_tab[sc];
    float f0[8], f1[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        f0[2 * j] = bf16_lo(w[j]);
        f0[2 * j + 1] = bf16_hi(w[j]);
        f1[2 * j] = bf16_lo(w[4 + j]);
        f1[2 * j + 1] = bf16_hi(w[4 + j]);
    }
    c0 = e2m1x8_encode(f0, enc);
    c1 = e2m1x8_encode(f1, enc);
    return sc;
}

// Byte offset of scale (row r, 16-element block kb) in the MMA scale layout:
// 512-byte atoms of 128 rows x 4 blocks, atoms K-fastest, `atoms_per_rowblk`
// atoms per 128-row block; inside an atom, row r sits at (r%32)*16 +
// ((r%128)/32)*4 and block kb at kb%4.
__host__ __device__ __forceinline__ int64_t sf_offset(int64_t r, int64_t kb, int64_t atoms_per_rowblk)
{
    return ((r >> 7) * atoms_per_rowblk + (kb >> 2)) * 512 + (r & 31) * 16 + ((r & 127) >> 5) * 4 + (kb & 3);
}

}  // namespace mq
