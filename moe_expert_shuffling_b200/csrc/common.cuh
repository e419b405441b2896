// Device helpers shared by the shuffle kernels (sm_100a): bulk async copies between
// global and shared memory tracked by mbarriers, bounded waits, and warp utilities.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "moe_shuffle.h"

namespace moe {

// A device wait gives up after this long and reports MOE_ERR_TIMEOUT instead of hanging.
constexpr uint64_t kWaitLimitNs = 1000ull * 1000ull * 1000ull;  // 1 s

__device__ __forceinline__ uint32_t smem_addr(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
                 : "memory");
}

// Make mbarrier initialisation visible to the async (bulk copy) proxy.
__device__ __forceinline__ void mbar_init_fence()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

// Wait for phase `parity` of `bar`; false if it did not complete within kWaitLimitNs.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 1; it < (1u << 30); ++it) {
        if (mbar_try_wait(bar, parity))
            return true;
        if ((it & 63u) == 0 && global_timer_ns() - t0 > kWaitLimitNs)
            return false;
    }
    return false;
}

// Bulk copy global -> shared; completion is counted on `bar` (transaction bytes).
// Both addresses 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_load(void *dst_smem, const void *src, uint32_t bytes,
                                          uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_addr(dst_smem)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

// Bulk copy shared -> global in the issuing thread's current bulk group.
__device__ __forceinline__ void bulk_store(void *dst, const void *src_smem, uint32_t bytes)
{
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst),
                 "r"(smem_addr(src_smem)), "r"(bytes)
                 : "memory");
}

// Order earlier shared-memory accesses before later async-proxy (bulk copy) accesses.
__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void bulk_commit()
{
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// Wait until at most N of this thread's bulk groups still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read()
{
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void bulk_wait_read_dyn(int n)
{
    // wait_group takes an immediate; cover the small lags the kernels use.
    switch (n) {
    case 0: bulk_wait_read<0>(); break;
    case 1: bulk_wait_read<1>(); break;
    case 2: bulk_wait_read<2>(); break;
    case 3: bulk_wait_read<3>(); break;
    case 4: bulk_wait_read<4>(); break;
    case 5: bulk_wait_read<5>(); break;
    case 6: bulk_wait_read<6>(); break;
    default: bulk_wait_read<7>(); break;
    }
}

__device__ __forceinline__ void bulk_wait_all()
{
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

__device__ __forceinline__ uint32_t lanemask_lt()
{
    uint32_t m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// 16-byte global load that does not allocate in L1 (each byte is read once).
__device__ __forceinline__ uint4 ld_stream_v4(const void *p)
{
    uint4 v;
    asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ void st_stream_v4(void *p, uint4 v)
{
    asm volatile("st.global.cs.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ uint4 lds_v4(const void *p)
{
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(smem_addr(p)));
    return v;
}

// Programmatic dependent launch.  A kernel launched with programmatic stream serialization
// may begin while the kernel before it on the stream is still finishing.  pdl_wait() returns
// once every earlier grid on the stream has completed and its memory operations are visible;
// every thread calls it before its first access to global memory (which an earlier kernel
// may still be writing, or still be reading).  pdl_trigger() lets the next kernel on the
// stream begin launching; it still waits for this grid to complete before its own global
// accesses.  Both do nothing in a kernel launched without the attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void pdl_trigger()
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// gpu-scope acquire / release accesses for flags and counters shared between CTAs.
__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t *a)
{
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(a) : "memory");
    return v;
}

__device__ __forceinline__ uint32_t atom_add_acq_rel_gpu(uint32_t *a, uint32_t v)
{
    uint32_t old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(a), "r"(v)
                 : "memory");
    return old;
}

__device__ __forceinline__ void st_release_gpu(uint32_t *a, uint32_t v)
{
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(a), "r"(v) : "memory");
}

// Order this thread's async-proxy (bulk copy) accesses to global memory against its
// generic-proxy accesses: after bulk stores have completed and before a flag is released;
// after a flag has been acquired and before bulk loads read what it guards.
__device__ __forceinline__ void fence_proxy_async_global()
{
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Relaxed read of a word that other CTAs may set (an error flag polled inside a wait).
__device__ __forceinline__ uint32_t ld_relaxed_gpu(const uint32_t *a)
{
    uint32_t v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(a) : "memory");
    return v;
}

// Sense-reversing grid barrier for a co-resident grid.  sync[0] counts arrivals; the last
// CTA to arrive sets it back to 0 and advances the generation word sync[1], which the
// others wait on, so the words are ready for the next barrier (and the next launch) with no
// extra step.  A wait gives up after kWaitLimitNs, sets MOE_ERR_TIMEOUT and returns false.
// All threads must call.
// `gen` is the generation read (by thread 0) before this CTA's phase began: it cannot
// advance until this CTA arrives, and reading it early takes a round trip off the barrier.
__device__ __forceinline__ bool grid_barrier(uint32_t *sync, uint32_t *err, uint32_t gen, int *s_ok)
{
    __syncthreads();
    if (threadIdx.x == 0) {
        bool ok = true;
        if (atom_add_acq_rel_gpu(&sync[0], 1u) == gridDim.x - 1u) {
            sync[0] = 0u;                // no CTA reads the count until the next barrier
            st_release_gpu(&sync[1], gen + 1u);
        } else {
            const uint64_t t0 = global_timer_ns();
            for (uint32_t it = 0; ld_acquire_gpu(&sync[1]) == gen; ++it) {
                if ((it & 15u) == 15u &&
                    (global_timer_ns() - t0 > kWaitLimitNs || it > (1u << 30))) {
                    atomicOr(err, MOE_ERR_TIMEOUT);
                    ok = false;
                    break;
                }
                __nanosleep(32);
            }
        }
        *s_ok = ok;
    }
    __syncthreads();
    return *s_ok != 0;
}

// Wait (one whole warp) until words[0..n) all hold `want` -- the arrival words that the CTAs
// or groups of a grid release (the group plan kernel).  Relaxed loads, all in flight at once,
// then one acquire fence.  Returns the same value in every lane; false after kWaitLimitNs
// (MOE_ERR_TIMEOUT set).
__device__ __forceinline__ bool wait_words_warp(const uint32_t *words, uint32_t n, uint32_t want,
                                                uint32_t *err)
{
    const uint32_t lane = threadIdx.x & 31u;
    bool ok = true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 0;; ++it) {
        bool mine = true;
        for (uint32_t q = lane; q < n; q += 32)
            mine &= ld_relaxed_gpu(words + q) == want;
        if (__all_sync(0xffffffffu, mine))
            break;
        if ((it & 15u) == 15u) {
            const bool late = global_timer_ns() - t0 > kWaitLimitNs || it > (1u << 30);
            if (__shfl_sync(0xffffffffu, late, 0)) {
                if (lane == 0)
                    atomicOr(err, MOE_ERR_TIMEOUT);
                ok = false;
                break;
            }
        }
    }
    // what each arrival released is visible to this CTA from here on
    asm volatile("fence.acq_rel.gpu;" ::: "memory");
    return ok;
}

// wait_words_warp run by warp 0, the result shared with the CTA.  All threads must call.
__device__ __forceinline__ bool wait_words(const uint32_t *words, uint32_t n, uint32_t want,
                                           uint32_t *err, int *s_ok)
{
    if (threadIdx.x < 32) {
        const bool ok = wait_words_warp(words, n, want, err);
        if (threadIdx.x == 0)
            *s_ok = ok;
    }
    __syncthreads();
    return *s_ok != 0;
}

__host__ __device__ constexpr int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
__host__ __device__ constexpr int64_t round_up(int64_t a, int64_t b) { return ceil_div(a, b) * b; }

}  // namespace moe
