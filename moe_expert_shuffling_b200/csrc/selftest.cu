// moe_wait_selftest: runs the library's bounded device waits on something that never
// completes, so that a caller (or a test) can see them give up and report MOE_ERR_TIMEOUT
// with the CUDA context still usable.  Nothing on the shuffle path calls it.
#include <cuda_runtime.h>

#include "combine_cta.cuh"
#include "common.cuh"
#include "internal.cuh"

namespace moe {
namespace {

// which = 0: the ready-flag wait of the fused kernel, on a flag nothing sets.
// which = 1: the mbarrier wait of the copy pipelines, on a barrier that expects two
//            arrivals and gets one (no copy is in flight).
// which = 2: the plan's grid barrier, in a grid of two CTAs of which only CTA 0 arrives.
// which = 3: the group plan's exchange wait, on two arrival words of which nothing sets
//            the second.
__global__ void wait_selftest_kernel(uint32_t *words, uint32_t *err, int which)
{
    __shared__ uint64_t bar;
    __shared__ int s_ok;
    const uint32_t *never_set = words;
    if (which == 2) {
        if (blockIdx.x == 0)
            (void)grid_barrier(words, err, 0u, &s_ok);  // words[0..1]: count, generation
        return;
    }
    if (which == 3) {
        if (blockIdx.x == 0) {
            if (threadIdx.x == 0)
                st_release_gpu(&words[0], 1u);  // the first group arrives, the second never
            (void)wait_words(words, 2u, 1u, err, &s_ok);
        }
        return;
    }
    if (blockIdx.x != 0)
        return;
    if (which == 0) {
        if (threadIdx.x == 0 && !wait_flag(never_set, 1u, err))
            atomicOr(err, MOE_ERR_TIMEOUT);
        return;
    }
    if (threadIdx.x == 0) {
        mbar_init(&bar, 2);
        mbar_init_fence();
    }
    __syncthreads();
    if (threadIdx.x == 0)
        mbar_arrive(&bar);
    const bool ok = mbar_wait_bounded(&bar, 0u);
    if (!__all_sync(0xffffffffu, ok) && threadIdx.x == 0)
        atomicOr(err, MOE_ERR_TIMEOUT);
}

}  // namespace

cudaError_t run_wait_selftest(int which, cudaStream_t stream, uint32_t *flags)
{
    // [0..1]: the flag nothing sets / the barrier's count and generation, [2]: error word
    uint32_t *words = nullptr;
    cudaError_t e = cudaMalloc(&words, 3 * sizeof(uint32_t));
    if (e != cudaSuccess)
        return e;
    e = cudaMemsetAsync(words, 0, 3 * sizeof(uint32_t), stream);
    if (e == cudaSuccess) {
        wait_selftest_kernel<<<2, 32, 0, stream>>>(words, words + 2, which);
        e = cudaGetLastError();
    }
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(flags, words + 2, sizeof(uint32_t), cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess)
        e = cudaStreamSynchronize(stream);
    const cudaError_t f = cudaFree(words);
    return e != cudaSuccess ? e : f;
}

}  // namespace moe
