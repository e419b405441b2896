// One warp's dispatch pipeline, shared by the dispatch kernel and the fused
// dispatch-and-combine kernel.
//
// recv[slot[t, j]] = x[t] for every routed entry (FUSCO, arXiv 2512.22036, abstract: the
// layout transformation happens as the data moves).  A unit is (token, row chunk).  Lane 0
// stages a chunk of x[t] into a ring stage with one bulk copy (cp.async.bulk, completion on
// the stage's mbarrier); once it has landed, lane j issues the bulk store of that chunk to
// receive row slot[t, j].  Every token row is read once and written k times.  A stage is
// refilled only after the stores that read it have drained (wait_group.read).
#pragma once

#include <algorithm>

#include "common.cuh"

namespace moe {

constexpr uint32_t kDispatchMaxChunkBytes = 32768;
constexpr int kDispatchMaxStages = 8;

// How a row is cut into units and laid out in a ring stage.
struct DispatchGeometry {
    uint32_t nchunks, chunk, scale_off, stage_bytes;
    bool bulk_scales;  // the scale row rides in the stage (its size is a multiple of 16 B)
};

// `min_chunks` asks for at least that many chunks per row (a decode-sized batch spreads its
// rows over more warps); chunks stay at least kDispatchMinChunkBytes.
constexpr uint32_t kDispatchMinChunkBytes = 2048;

inline DispatchGeometry dispatch_geometry(uint32_t row_bytes, uint32_t srow_bytes,
                                          uint32_t min_chunks = 1)
{
    DispatchGeometry g;
    uint32_t n = static_cast<uint32_t>(ceil_div(row_bytes, kDispatchMaxChunkBytes));
    const uint32_t most = static_cast<uint32_t>(
        std::max<int64_t>(1, row_bytes / kDispatchMinChunkBytes));
    if (min_chunks > n)
        n = std::min(min_chunks, std::max(n, most));
    g.chunk = static_cast<uint32_t>(round_up(ceil_div(row_bytes, n), 16));
    g.nchunks = static_cast<uint32_t>(ceil_div(row_bytes, g.chunk));
    g.bulk_scales = srow_bytes > 0 && srow_bytes % 16 == 0;
    g.scale_off = static_cast<uint32_t>(round_up(g.chunk, 128));
    g.stage_bytes =
        static_cast<uint32_t>(round_up(g.scale_off + (g.bulk_scales ? srow_bytes : 0u), 128));
    return g;
}

struct DispatchParams {
    const uint8_t *x;
    const uint8_t *xs;
    uint8_t *recv;
    uint8_t *rs;
    const int32_t *slot;
    uint32_t *err;
    uint32_t units;         // N * nchunks (< 2^31)
    uint32_t per_warp;      // units of each warp: [warp * per_warp, +per_warp)
    int32_t k, n_rows;
    uint32_t nchunks;
    int32_t stages, lag;
    uint32_t row_bytes, srow_bytes, chunk_bytes, stage_bytes, scale_off, bar_bytes;
    bool bulk_scales;
};

// The warp's ring: `stages` mbarriers (initialised with count 1) and as many stages of
// p.stage_bytes.  Units [u0, u0 + n) go through it; `seq` is the number of units the ring
// has carried before, so that stage indices and mbarrier phases continue across runs.
// Returns false (MOE_ERR_TIMEOUT set) if a load did not land within the wait limit.  On
// return every store of the run has finished reading shared memory; with `complete` the
// stores have also completed (their data is in global memory).
__device__ __forceinline__ bool dispatch_warp_run(const DispatchParams &p, uint64_t *bars,
                                                  uint8_t *stage0, uint32_t u0, int n,
                                                  uint32_t seq, bool complete)
{
    const int lane = threadIdx.x & 31;
    const int S = p.stages;

    // Issue the load of the run's i-th unit into its stage (lane 0 only).
    auto issue_load = [&](int i) {
        const uint32_t u = u0 + static_cast<uint32_t>(i);
        const uint32_t t = u / p.nchunks;
        const uint32_t c = u - t * p.nchunks;
        const uint32_t off = c * p.chunk_bytes;
        const uint32_t len = min(p.chunk_bytes, p.row_bytes - off);
        const int s = static_cast<int>((seq + static_cast<uint32_t>(i)) % S);
        uint8_t *st = stage0 + static_cast<size_t>(s) * p.stage_bytes;
        const bool sc = p.bulk_scales && c == 0;
        mbar_arrive_expect_tx(&bars[s], len + (sc ? p.srow_bytes : 0u));
        bulk_load(st, p.x + static_cast<int64_t>(t) * p.row_bytes + off, len, &bars[s]);
        if (sc)
            bulk_load(st + p.scale_off, p.xs + static_cast<int64_t>(t) * p.srow_bytes,
                      p.srow_bytes, &bars[s]);
    };

    int next_load = S < n ? S : n;  // units [0, next_load) have been issued
    if (lane == 0)
        for (int i = 0; i < next_load; ++i)
            issue_load(i);

    int32_t cur = -1;
    if (n > 0 && lane < p.k)
        cur = __ldg(p.slot + (u0 / p.nchunks) * p.k + lane);

    bool ok = true;
    int i = 0;
    for (; i < n; ++i) {
        const uint32_t q = seq + static_cast<uint32_t>(i);
        const int s = static_cast<int>(q % S);
        const uint32_t parity = (q / S) & 1u;
        const uint32_t u = u0 + static_cast<uint32_t>(i);
        const uint32_t t = u / p.nchunks;
        const uint32_t c = u - t * p.nchunks;
        const uint32_t off = c * p.chunk_bytes;
        const uint32_t len = min(p.chunk_bytes, p.row_bytes - off);

        // Slots of the next unit, fetched while this unit's row is in flight.
        int32_t nxt = -1;
        if (i + 1 < n && lane < p.k)
            nxt = __ldg(p.slot + ((u + 1) / p.nchunks) * p.k + lane);

        const bool landed = mbar_wait_bounded(&bars[s], parity);
        if (!__all_sync(0xffffffffu, landed)) {
            ok = false;
            break;
        }
        fence_proxy_async_smem();
        const uint8_t *st = stage0 + static_cast<size_t>(s) * p.stage_bytes;
        if (lane < p.k && static_cast<uint32_t>(cur) < static_cast<uint32_t>(p.n_rows)) {
            bulk_store(p.recv + static_cast<int64_t>(cur) * p.row_bytes + off, st, len);
            if (p.bulk_scales && c == 0)
                bulk_store(p.rs + static_cast<int64_t>(cur) * p.srow_bytes, st + p.scale_off,
                           p.srow_bytes);
        }
        bulk_commit();

        // Refill the stage of unit i - lag once its stores have read shared memory.
        const int r = i - p.lag;
        if (r >= 0 && r + S < n) {
            bulk_wait_read_dyn(p.lag);
            __syncwarp();
            if (lane == 0)
                issue_load(r + S);
            next_load = r + S + 1;
        }
        cur = nxt;
    }
    if (complete)
        bulk_wait_all();
    else
        bulk_wait_read<0>();
    if (!ok) {
        if (lane == 0)
            atomicOr(p.err, MOE_ERR_TIMEOUT);
        // Let loads still in flight land before the ring is reused or released.
        for (int m = i; m < next_load; ++m) {
            const uint32_t q = seq + static_cast<uint32_t>(m);
            (void)mbar_wait_bounded(&bars[q % S], (q / S) & 1u);
        }
    }
    __syncwarp();
    return ok;
}

}  // namespace moe
