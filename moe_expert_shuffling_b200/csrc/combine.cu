// Combine: out[t] = bf16_rne( fp32 fma chain over j = 0..k-1 of w[t, j] * y[slot[t, j]] ),
// starting from +0 -- the expert results of a token brought back and summed (DySHARP blog,
// sections 1-2).  The chain runs in top-k column order, so every launch configuration
// gives the same bits.
//
// Engine: a persistent grid of warps over work units (token, column chunk of 32*VPL
// 16-byte vectors).  A warp reads the token's k slots and weights once (lane j holds
// column j), then each lane issues all of its KB x VPL row loads before the first fma,
// so up to KB*VPL 16-byte loads per lane are in flight.  Loads bypass L1 (each byte of
// y is read once); the output vector is written once with a streaming store.
#include <algorithm>

#include <cuda_bf16.h>

#include "common.cuh"
#include "internal.cuh"

namespace moe {
namespace {

constexpr int kCombineThreads = 256;
constexpr uint32_t kFull = 0xffffffffu;

struct CombineParams {
    const uint16_t *y;
    const int32_t *slot;
    const float *w;
    uint16_t *out;
    uint32_t units;         // N * nchunks (< 2^31)
    int32_t N, k, n_rows, H, nvec;
    uint32_t nchunks;
};

__device__ __forceinline__ void fma_bf16x8(float *acc, float wj, const uint4 &v)
{
    const uint32_t words[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const float lo = __uint_as_float(words[q] << 16);
        const float hi = __uint_as_float(words[q] & 0xffff0000u);
        acc[2 * q] = __fmaf_rn(wj, lo, acc[2 * q]);
        acc[2 * q + 1] = __fmaf_rn(wj, hi, acc[2 * q + 1]);
    }
}

__device__ __forceinline__ uint4 pack_bf16x8(const float *acc)
{
    uint32_t words[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(acc[2 * q], acc[2 * q + 1]);
        words[q] = *reinterpret_cast<const uint32_t *>(&h);
    }
    return make_uint4(words[0], words[1], words[2], words[3]);
}

template <int KB, int VPL>
__global__ void __launch_bounds__(kCombineThreads) combine_kernel(const CombineParams p)
{
    const int lane = threadIdx.x & 31;
    const uint32_t gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const uint32_t nw = (gridDim.x * blockDim.x) >> 5;

    for (uint32_t u = gw; u < p.units; u += nw) {
        const uint32_t t = u / p.nchunks;
        const int c = static_cast<int>(u - t * p.nchunks);
        int32_t my_s = -1;
        float my_w = 0.f;
        if (lane < p.k) {
            my_s = __ldg(p.slot + static_cast<int64_t>(t) * p.k + lane);
            my_w = __ldg(p.w + static_cast<int64_t>(t) * p.k + lane);
        }
        float acc[VPL][8];
#pragma unroll
        for (int q = 0; q < VPL; ++q)
#pragma unroll
            for (int i = 0; i < 8; ++i)
                acc[q][i] = 0.f;
        const int v0 = c * (32 * VPL) + lane;

        for (int j0 = 0; j0 < p.k; j0 += KB) {
            uint4 v[KB][VPL];
#pragma unroll
            for (int jj = 0; jj < KB; ++jj) {
                const int j = j0 + jj;
                const int32_t s = __shfl_sync(kFull, my_s, j & 31);
                const bool ok =
                    j < p.k && static_cast<uint32_t>(s) < static_cast<uint32_t>(p.n_rows);
                const uint16_t *row = p.y + static_cast<int64_t>(ok ? s : 0) * p.H;
#pragma unroll
                for (int q = 0; q < VPL; ++q) {
                    const int vec = v0 + q * 32;
                    v[jj][q] = (ok && vec < p.nvec) ? ld_stream_v4(row + static_cast<int64_t>(vec) * 8)
                                                    : make_uint4(0u, 0u, 0u, 0u);
                }
            }
#pragma unroll
            for (int jj = 0; jj < KB; ++jj) {
                const int j = j0 + jj;
                const int32_t s = __shfl_sync(kFull, my_s, j & 31);
                const float wj = __shfl_sync(kFull, my_w, j & 31);
                if (j < p.k && static_cast<uint32_t>(s) < static_cast<uint32_t>(p.n_rows)) {
#pragma unroll
                    for (int q = 0; q < VPL; ++q)
                        fma_bf16x8(acc[q], wj, v[jj][q]);
                }
            }
        }
        uint16_t *orow = p.out + static_cast<int64_t>(t) * p.H;
#pragma unroll
        for (int q = 0; q < VPL; ++q) {
            const int vec = v0 + q * 32;
            if (vec < p.nvec)
                st_stream_v4(orow + static_cast<int64_t>(vec) * 8, pack_bf16x8(acc[q]));
        }
    }
}

template <int KB, int VPL>
cudaError_t launch_one(const CombineParams &p, int device, int ctas_per_sm, cudaStream_t stream)
{
    auto kern = combine_kernel<KB, VPL>;
    int per_sm = 0;
    cudaError_t e =
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kCombineThreads, 0);
    if (e != cudaSuccess)
        return e;
    per_sm = std::max(per_sm, 1);
    if (ctas_per_sm > 0)
        per_sm = std::min(per_sm, ctas_per_sm);
    const int64_t warps_per_cta = kCombineThreads / 32;
    const int64_t grid = std::max<int64_t>(
        1, std::min<int64_t>(ceil_div(p.units, warps_per_cta),
                             static_cast<int64_t>(sm_count(device)) * per_sm));
    kern<<<static_cast<unsigned>(grid), kCombineThreads, 0, stream>>>(p);
    return cudaGetLastError();
}

template <int KB>
cudaError_t launch_kb(const CombineParams &p, int vpl, int device, int ctas, cudaStream_t s)
{
    switch (vpl) {
    case 1: return launch_one<KB, 1>(p, device, ctas, s);
    case 4: return launch_one<KB, 4>(p, device, ctas, s);
    default: return launch_one<KB, 2>(p, device, ctas, s);
    }
}

}  // namespace

cudaError_t launch_combine(const CombineArgs &a, int device, cudaStream_t stream)
{
    if (a.N == 0)
        return cudaSuccess;
    const Tuning &tu = tuning();
    int vpl = tu.combine_vec_per_lane > 0 ? tu.combine_vec_per_lane : 1;
    if (vpl != 1 && vpl != 2 && vpl != 4)
        vpl = 1;
    CombineParams p;
    p.y = a.y;
    p.slot = a.slot;
    p.w = a.w;
    p.out = a.out;
    p.N = a.N;
    p.k = a.k;
    p.n_rows = a.n_rows;
    p.H = a.H;
    p.nvec = a.H / 8;
    p.nchunks = static_cast<uint32_t>(ceil_div(p.nvec, 32 * vpl));
    const int64_t units = static_cast<int64_t>(a.N) * p.nchunks;
    if (units >= (int64_t(1) << 31))
        return cudaErrorInvalidValue;
    p.units = static_cast<uint32_t>(units);
    const int ctas = tu.combine_ctas_per_sm;
    if (a.k <= 2)
        return launch_kb<2>(p, vpl, device, ctas, stream);
    if (a.k <= 4)
        return launch_kb<4>(p, vpl, device, ctas, stream);
    return launch_kb<8>(p, vpl, device, ctas, stream);
}

}  // namespace moe
