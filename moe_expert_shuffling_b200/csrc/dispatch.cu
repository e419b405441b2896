// Dispatch: recv[slot[t, j]] = x[t] for every routed entry, with the expert-major layout
// produced by the copy itself (FUSCO, arXiv 2512.22036, abstract; FUSCO summary, Group 3:
// data is placed at its destination with no staging buffer and no later rearrangement).
//
// Engine: warps each running their own bulk-copy pipeline (dispatch_warp.cuh) over a
// contiguous run of work units (token, row chunk), so every token row is read from HBM
// once and written k times -- the "read once, fan out locally" form of FUSCO's dedup (one
// move per token, which is at most one per destination rank).  fp8 rows carry their fp32
// scale block along when its size is a multiple of 16 bytes; otherwise a small second
// kernel moves the scales.
#include <algorithm>

#include "common.cuh"
#include "dispatch_warp.cuh"
#include "internal.cuh"

namespace moe {
namespace {

// Measured on B200 (dsv3 and long shapes): short runs of 2 units per warp on a grid that
// covers all units beat persistent warps by ~12% (the block scheduler evens out the
// tail); 4 stages with 2 store groups in flight per warp.
constexpr int kDefaultUnitsPerWarp = 2;
constexpr int64_t kSplitUnitsPerSm = 4;

__global__ void __launch_bounds__(128) dispatch_bulk_kernel(const DispatchParams p)
{
    extern __shared__ __align__(128) uint8_t smem[];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, wpc = blockDim.x >> 5;
    const int S = p.stages;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem) + wid * S;
    uint8_t *stage0 = smem + p.bar_bytes + static_cast<size_t>(wid) * S * p.stage_bytes;

    const uint32_t gw = blockIdx.x * wpc + wid;
    const uint32_t u0 = gw * p.per_warp;  // this warp's first unit
    const int n_my = u0 < p.units ? static_cast<int>(min(p.per_warp, p.units - u0)) : 0;

    if (lane == 0) {
        for (int s = 0; s < S; ++s)
            mbar_init(&bars[s], 1);
        mbar_init_fence();
    }
    pdl_trigger();
    pdl_wait();  // the plan's slots and the payload are read from here on
    __syncwarp();
    (void)dispatch_warp_run(p, bars, stage0, u0, n_my, 0u, true);
}

// Scale rows whose size is not a multiple of 16 bytes: one thread per fp32 scale.
__global__ void dispatch_scales_kernel(const float *__restrict__ xs, float *__restrict__ rs,
                                       const int32_t *__restrict__ slot, int64_t entries,
                                       int32_t k, int32_t ncols, int32_t n_rows)
{
    pdl_trigger();
    pdl_wait();
    const int64_t total = entries * ncols;
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t ent = i / ncols;
        const int32_t c = static_cast<int32_t>(i - ent * ncols);
        const int32_t s = slot[ent];
        if (static_cast<uint32_t>(s) < static_cast<uint32_t>(n_rows))
            rs[static_cast<int64_t>(s) * ncols + c] = xs[(ent / k) * ncols + c];
    }
}

}  // namespace

cudaError_t launch_dispatch(const DispatchArgs &a, int device, cudaStream_t stream)
{
    if (a.N == 0)
        return cudaSuccess;
    const Tuning &tu = tuning();
    int stages = tu.dispatch_stages > 0 ? tu.dispatch_stages : 4;
    stages = std::min(std::max(stages, 2), kDispatchMaxStages);
    int lag = tu.dispatch_lag > 0 ? tu.dispatch_lag : 2;
    lag = std::min(std::max(lag, 1), std::min(stages - 1, 7));
    int wpc = tu.dispatch_warps_per_cta > 0 ? tu.dispatch_warps_per_cta : 1;
    wpc = std::min(std::max(wpc, 1), 4);

    // Few tokens (a decode-sized batch): cut the rows into more chunks, so that there are
    // about kSplitUnitsPerSm (token, chunk) units per SM rather than a handful of warps each
    // moving whole rows.
    DispatchGeometry g = dispatch_geometry(a.row_bytes, a.srow_bytes);
    const int64_t split_units = tu.dispatch_split_units == 1 ? 0
                                : tu.dispatch_split_units > 1
                                    ? tu.dispatch_split_units
                                    : static_cast<int64_t>(sm_count(device)) * kSplitUnitsPerSm;
    if (static_cast<int64_t>(a.N) * g.nchunks < split_units)
        g = dispatch_geometry(a.row_bytes, a.srow_bytes,
                              static_cast<uint32_t>(std::min<int64_t>(
                                  ceil_div(split_units, a.N), 1 << 16)));
    const uint32_t nchunks = g.nchunks, chunk = g.chunk, scale_off = g.scale_off,
                   stage_bytes = g.stage_bytes;
    const bool bulk_scales = g.bulk_scales;

    const int max_optin = max_smem_optin(device);
    cudaError_t e = cudaSuccess;
    auto smem_for = [&](int st) {
        return static_cast<size_t>(round_up(static_cast<int64_t>(wpc) * st * 8, 128)) +
               static_cast<size_t>(wpc) * st * stage_bytes;
    };
    while (stages > 2 && smem_for(stages) > static_cast<size_t>(max_optin))
        --stages;
    while (wpc > 1 && smem_for(stages) > static_cast<size_t>(max_optin))
        --wpc;
    if (smem_for(stages) > static_cast<size_t>(max_optin))
        return cudaErrorInvalidValue;
    lag = std::min(lag, stages - 1);
    const size_t smem = smem_for(stages);

    int per_sm = 0;
    e = kernel_fit(reinterpret_cast<const void *>(dispatch_bulk_kernel), device, wpc * 32, smem,
                   &per_sm);
    if (e != cudaSuccess)
        return e;
    if (per_sm < 1)
        return cudaErrorInvalidConfiguration;
    if (tu.dispatch_ctas_per_sm > 0)
        per_sm = std::min(per_sm, tu.dispatch_ctas_per_sm);

    DispatchParams p;
    p.x = a.x;
    p.xs = a.xs;
    p.recv = a.recv;
    p.rs = a.rs;
    p.slot = a.slot;
    p.err = a.err;
    const int64_t units = static_cast<int64_t>(a.N) * nchunks;
    if (units >= (int64_t(1) << 31))
        return cudaErrorInvalidValue;
    p.units = static_cast<uint32_t>(units);
    p.k = a.k;
    p.n_rows = a.n_rows;
    p.nchunks = nchunks;
    p.stages = stages;
    p.lag = lag;
    p.row_bytes = a.row_bytes;
    p.srow_bytes = a.srow_bytes;
    p.chunk_bytes = chunk;
    p.stage_bytes = stage_bytes;
    p.scale_off = scale_off;
    p.bar_bytes = static_cast<uint32_t>(round_up(static_cast<int64_t>(wpc) * stages * 8, 128));
    p.bulk_scales = bulk_scales;

    // Each warp takes a contiguous run of units; the grid covers all of them, so CTAs
    // that finish early are replaced by the block scheduler (balances the tail).
    const int64_t resident_warps = static_cast<int64_t>(sm_count(device)) * per_sm * wpc;
    int64_t per_warp = tu.dispatch_units_per_warp > 0 ? tu.dispatch_units_per_warp
                                                      : kDefaultUnitsPerWarp;
    if (per_warp < 0 || ceil_div(units, per_warp) < resident_warps)
        per_warp = std::max<int64_t>(1, ceil_div(units, resident_warps));
    p.per_warp = static_cast<uint32_t>(per_warp);
    const int64_t grid = std::max<int64_t>(1, ceil_div(ceil_div(units, per_warp), wpc));
    e = launch_kernel(dispatch_bulk_kernel, dim3(static_cast<unsigned>(grid)), dim3(wpc * 32),
                      smem, stream, false, device, p);
    if (e != cudaSuccess)
        return e;

    if (a.srow_bytes > 0 && !bulk_scales) {
        const int32_t ncols = static_cast<int32_t>(a.srow_bytes / 4);
        const int64_t entries = static_cast<int64_t>(a.N) * a.k;
        const int64_t total = entries * ncols;
        const int64_t blocks = std::min<int64_t>(ceil_div(total, 256), sm_count(device) * 8);
        e = launch_kernel(dispatch_scales_kernel,
                          dim3(static_cast<unsigned>(std::max<int64_t>(blocks, 1))), dim3(256), 0,
                          stream, false, device, reinterpret_cast<const float *>(a.xs),
                          reinterpret_cast<float *>(a.rs), a.slot, entries,
                          static_cast<int32_t>(a.k), ncols, static_cast<int32_t>(a.n_rows));
    }
    return e;
}

}  // namespace moe
