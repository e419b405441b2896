// Dispatch and combine in one persistent launch (moe_dispatch_combine): the single-GPU form
// of DySHARP's token-centric kernel fusion (DySHARP blog, section 6: Dispatch and Combine
// of different tokens run at the same time inside one kernel, each starting as soon as its
// inputs are ready, instead of as two collective phases one after the other).
//
// Every CTA can do both kinds of work item:
//   dispatch item -- d_run_tokens tokens; each dispatch warp of the CTA takes its own items
//                    and runs them through its ring (dispatch_warp.cuh);
//   combine item  -- c_run_tokens tokens; the CTA's producer warp and consumer warps run
//                    them through the combine ring (combine_cta.cuh).
// Items are handed out by two global counters.  CTAs [0, d_first_ctas) take dispatch items
// until none is left and then combine items; the other CTAs do the reverse, so both kinds
// run side by side and whichever runs out first lends its CTAs to the other.
//
// When the combine reads the rows this launch dispatches (y == recv, one plan), token t is
// combined only after ready[t] holds this launch's epoch.  The warp that dispatched t sets
// it once the token's bulk stores have completed (wait_group 0, proxy fence, release); the
// combine producer acquires it and fences before its bulk loads.  The epoch lives in device
// memory (work[3] + 1, advanced by each launch's last CTA), so a launch replayed from a
// CUDA graph never sees the flags of an earlier replay as its own.  Dispatch work never
// waits on combine work and the grid is co-resident (cooperative launch), so every flag a
// combine waits on is set by a CTA that is running: no wait can deadlock.  Without flags no
// CTA waits on another, and the launch is an ordinary one.  Each wait still
// gives up after the wait limit, or as soon as another CTA reports a timeout, and the
// error word then carries MOE_ERR_TIMEOUT.
#include <algorithm>

#include "combine_cta.cuh"
#include "common.cuh"
#include "dispatch_warp.cuh"
#include "internal.cuh"

namespace moe {
namespace {

// Defaults, measured on B200 over the dsv3, skew, long, Mixtral, top-16 and top-32 shapes
// (independent expert outputs), and dsv3 and Mixtral with y = recv:
//  * 4 CTAs of 48 KB per SM for CW = 4 consumer warps; narrower chunks (CW = 2, 1) get
//    proportionally more, smaller CTAs, as the combine kernel does;
//  * dispatch items of about 64 KB of traffic, at least one token (1 token of the dsv3 shape,
//    2 of long context, 3 of Mixtral), or about 144 KB when the combine waits on flags (6
//    tokens of Mixtral: smaller items raise the flag traffic);
//  * combine items of about 512 KB of traffic, at most 4 tokens (half of both when they
//    wait on flags);
//  * 10% of the CTAs starting on dispatch (30% when the combine waits on flags: with fewer,
//    most CTAs would wait for the few that dispatch).
// With these the fused step takes 0.95-0.98x the time of the two separate kernels.
// The wide combine shape for k <= 4 (eight consumer warps, 4 KB per row) was measured on the
// Mixtral shape: 3 CTAs of 64 KB per SM, combine items of up to 4 tokens (also when they
// wait on flags) and 30% of the CTAs starting on dispatch; these defaults gave 76-80 us per
// step against 85-101 us for the narrower shape's defaults.
constexpr int kDefaultCtasPerSm = 4;
constexpr int kDefaultSmemKb = 48;
constexpr int kDefaultDispatchSharePct = 10;
constexpr int kDefaultDispatchSharePctFlags = 30;
constexpr int kWideCtasPerSm = 3;
constexpr int kWideSmemKb = 64;
constexpr int kWideDispatchSharePct = 30;
// Graph-replayed steps with 256 KB dispatch items against the current sizes: long context
// 857.6 -> 837.5 us, dsv3 639.5 -> 638.6, Mixtral 79.2 -> 75.6 (independent expert outputs)
// and 78.2 -> 74.1 us (y = recv, flags); top-32 unchanged (one token is already 473 KB).
constexpr double kDispatchItemBytes = 64.0 * 1024;
constexpr double kDispatchItemBytesFlags = 144.0 * 1024;
constexpr double kCombineItemBytes = 512.0 * 1024;
constexpr uint32_t kMaxCombineRun = 4;
constexpr int kDispatchStages = 4;

struct FusedParams {
    DispatchParams d;
    CombineBulkParams c;
    uint32_t *work;        // [4]: next dispatch item, next combine item, CTAs done, epoch
    uint32_t *ready;       // [ready_len] per-token flags of the dispatch plan
    uint32_t ready_len;
    bool use_flags;        // the combine reads the rows this launch dispatches
    uint32_t d_items, d_run_tokens, c_items, c_run_tokens;
    uint32_t d_first_ctas;
    int32_t d_warps;       // dispatch warps per CTA
    int32_t N_d;           // dispatched tokens
    uint32_t d_bar_off;    // byte offset of the dispatch mbarriers in shared memory
};

template <int KMAX, int CW, bool RANKED>
__global__ void __launch_bounds__(Shape<CW>::kThreads, 1)
    fused_dispatch_combine_kernel(const FusedParams fp)
{
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ uint32_t s_item, s_epoch;
    __shared__ int s_abort, s_last;
    volatile int *abort_flag = &s_abort;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const DispatchParams &dp = fp.d;
    const CombineBulkParams &cp = fp.c;
    pdl_trigger();
    pdl_wait();  // every global access of the launch follows the previous kernel on the stream

    // Shared memory: combine mbarriers | combine ring + rank tables, overlaid by the
    // dispatch warps' rings | dispatch mbarriers.  A CTA switches roles only after all of
    // its copies of the previous role have completed.
    CombineRing r;
    r.carve<RANKED>(cp, smem, warp);
    const bool d_warp = warp < fp.d_warps;
    const int dw = d_warp ? warp : 0;
    uint64_t *dbars = reinterpret_cast<uint64_t *>(smem + fp.d_bar_off) + dw * dp.stages;
    uint8_t *dstage0 = smem + cp.bar_bytes + static_cast<size_t>(dw) * dp.stages * dp.stage_bytes;
    if (threadIdx.x == 0) {
        r.init<CW>();
        *abort_flag = 0;
        s_epoch = *reinterpret_cast<volatile uint32_t *>(fp.work + 3) + 1u;
    }
    if (d_warp && lane == 0) {
        for (int s = 0; s < dp.stages; ++s)
            mbar_init(&dbars[s], 1);
        mbar_init_fence();
    }
    __syncthreads();

    const uint32_t epoch = s_epoch;
    const uint32_t *wait_on = fp.use_flags ? fp.ready : nullptr;
    uint32_t dseq = 0;  // units this warp's dispatch ring has carried
    int ci = 0;         // chunks through the combine ring (the same count in every warp)
    const bool d_first = blockIdx.x < fp.d_first_ctas;
    for (int phase = 0; phase < 2; ++phase) {
        if ((phase == 0) == d_first) {
            // ---------------- dispatch items, taken warp by warp
            if (d_warp) {
                for (;;) {
                    uint32_t item = fp.d_items;
                    if (lane == 0 && *abort_flag == 0)
                        item = atomicAdd(&fp.work[0], 1u);
                    item = __shfl_sync(0xffffffffu, item, 0);
                    if (item >= fp.d_items)
                        break;
                    const uint32_t t0 = item * fp.d_run_tokens;
                    const uint32_t nt = min(fp.d_run_tokens, static_cast<uint32_t>(fp.N_d) - t0);
                    const int n = static_cast<int>(nt * dp.nchunks);
                    const bool ok = dispatch_warp_run(dp, dbars, dstage0, t0 * dp.nchunks, n, dseq,
                                                      fp.use_flags);
                    dseq += static_cast<uint32_t>(n);
                    if (!ok) {
                        if (lane == 0) {
                            *abort_flag = 1;
                            atomicOr(cp.err, MOE_ERR_TIMEOUT);  // stop the combine's waits too
                        }
                        break;
                    }
                    if (fp.use_flags) {
                        // every store of the item has completed: publish its tokens
                        fence_proxy_async_global();
                        __threadfence();
                        __syncwarp();
                        if (static_cast<uint32_t>(lane) < nt)
                            st_release_gpu(fp.ready + t0 + lane, epoch);
                    }
                }
            }
        } else {
            // ---------------- combine items, taken by the whole CTA
            if (RANKED)
                for (int q = threadIdx.x; q <= cp.R; q += blockDim.x)
                    r.roff_s[q] = __ldg(cp.rank_off + q);
            for (;;) {
                if (threadIdx.x == 0)
                    s_item = *abort_flag ? fp.c_items : atomicAdd(&fp.work[1], 1u);
                __syncthreads();
                const uint32_t item = s_item;
                __syncthreads();
                if (item >= fp.c_items)
                    break;
                const uint32_t b = item * fp.c_run_tokens;
                const int n_tok =
                    static_cast<int>(min(fp.c_run_tokens, static_cast<uint32_t>(cp.N) - b));
                int32_t s_first = -1;
                float w_first = 0.f;
                if (lane < cp.k) {
                    s_first = __ldg(cp.slot + static_cast<int64_t>(b) * cp.k + lane);
                    if (warp > 0)
                        w_first = __ldg(cp.w + static_cast<int64_t>(b) * cp.k + lane);
                }
                const bool ok =
                    warp == 0 ? combine_produce<KMAX, CW, RANKED>(cp, r, b, n_tok, s_first, ci,
                                                                  wait_on, epoch)
                              : combine_consume<KMAX, CW, RANKED>(cp, r, b, n_tok, s_first,
                                                                  w_first, ci);
                if (!ok && lane == 0)
                    *abort_flag = 1;
            }
        }
        __syncthreads();
        fence_proxy_async_smem();  // the next role reuses the same shared memory
    }

    // The launch's last CTA sets the work counters back to zero and advances the epoch
    // for the next launch; before the epoch would wrap, it clears every flag instead.
    if (threadIdx.x == 0) {
        __threadfence();
        s_last = atomicAdd(&fp.work[2], 1u) == gridDim.x - 1u;
    }
    __syncthreads();
    if (s_last) {
        uint32_t next = epoch;
        if (next == 0xffffffffu) {
            for (uint32_t q = threadIdx.x; q < fp.ready_len; q += blockDim.x)
                fp.ready[q] = 0u;
            next = 0u;
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            fp.work[0] = 0u;
            fp.work[1] = 0u;
            fp.work[3] = next;
            __threadfence();
            fp.work[2] = 0u;
        }
    }
}

template <int KMAX, int CW, bool RANKED>
cudaError_t launch_fused_shape(const FusedArgs &a, int device, cudaStream_t stream)
{
    constexpr uint32_t chunk = Shape<CW>::kChunk;
    constexpr int threads = Shape<CW>::kThreads;
    const Tuning &tu = tuning();
    const int max_optin = max_smem_optin(device);

    FusedParams fp{};
    fp.work = a.work;
    fp.ready = a.ready;
    fp.ready_len = a.ready_len;
    fp.use_flags = a.use_flags;
    fp.N_d = a.d.N;

    // dispatch side
    const DispatchGeometry g = dispatch_geometry(a.d.row_bytes, a.d.srow_bytes);
    if (a.d.srow_bytes > 0 && !g.bulk_scales)
        return cudaErrorInvalidValue;
    const int64_t d_units = static_cast<int64_t>(a.d.N) * g.nchunks;
    if (d_units >= (int64_t(1) << 31))
        return cudaErrorInvalidValue;
    DispatchParams &d = fp.d;
    d.x = a.d.x;
    d.xs = a.d.xs;
    d.recv = a.d.recv;
    d.rs = a.d.rs;
    d.slot = a.d.slot;
    d.err = a.d.err;
    d.units = static_cast<uint32_t>(d_units);
    d.per_warp = 0;
    d.k = a.d.k;
    d.n_rows = a.d.n_rows;
    d.nchunks = g.nchunks;
    d.row_bytes = a.d.row_bytes;
    d.srow_bytes = a.d.srow_bytes;
    d.chunk_bytes = g.chunk;
    d.stage_bytes = g.stage_bytes;
    d.scale_off = g.scale_off;
    d.bar_bytes = 0;
    d.bulk_scales = g.bulk_scales;

    // combine side
    CombineBulkParams &c = fp.c;
    c.y = reinterpret_cast<const uint8_t *>(a.c.y);
    c.slot = a.c.slot;
    c.w = a.c.w;
    c.out = reinterpret_cast<uint8_t *>(a.c.out);
    c.err = a.c.err;
    c.N = a.c.N;
    c.k = a.c.k;
    c.n_rows = a.c.n_rows;
    c.row_bytes = static_cast<uint32_t>(a.c.H) * 2u;
    c.nchunks = static_cast<uint32_t>(ceil_div(c.row_bytes, chunk));
    c.stage_bytes = static_cast<uint32_t>(a.c.k) * chunk;
    c.per_cta = 0;
    c.csplit = 1;
    c.rank_off = a.c.rank_off;
    c.R = a.c.R;

    // Shared memory: as many 4-stage dispatch rings as the budget holds (at least one,
    // with fewer stages if even one does not fit), and a combine ring using the larger of
    // the budget and the dispatch rings' area.
    constexpr bool kWide = CW >= 8;
    const size_t budget = static_cast<size_t>(
        std::min((tu.fused_smem_kb > 0 ? tu.fused_smem_kb
                                       : kWide ? kWideSmemKb : kDefaultSmemKb * CW / 4) *
                     1024,
                 max_optin));
    int d_stages = kDispatchStages;
    while (d_stages > 2 && static_cast<size_t>(d_stages) * g.stage_bytes > budget)
        --d_stages;
    const int d_warps = static_cast<int>(std::min<size_t>(
        1 + CW, std::max<size_t>(1, budget / (static_cast<size_t>(d_stages) * g.stage_bytes))));
    d.stages = d_stages;
    d.lag = std::min(2, d_stages - 1);
    const size_t d_area = static_cast<size_t>(d_warps) * d_stages * g.stage_bytes;
    const size_t tables =
        RANKED ? sizeof(int32_t) * (static_cast<size_t>(a.c.R) + 1 + 64 * CW) : 0;
    const size_t area = std::max(budget, d_area);
    int S = static_cast<int>(area > tables ? (area - tables) / c.stage_bytes : 0);
    S = std::max(2, std::min(S, kMaxBulkStages));
    c.stages = static_cast<uint32_t>(S);
    c.bar_bytes = static_cast<uint32_t>(round_up(2 * S * 8, 128));
    c.ring_bytes = static_cast<uint32_t>(S) * c.stage_bytes;
    const size_t c_area = c.ring_bytes + tables;
    fp.d_bar_off = static_cast<uint32_t>(
        c.bar_bytes + round_up(static_cast<int64_t>(std::max(c_area, d_area)), 128));
    const size_t smem =
        fp.d_bar_off + static_cast<size_t>(round_up(static_cast<int64_t>(d_warps) * d_stages * 8, 128));
    if (smem > static_cast<size_t>(max_optin))
        return cudaErrorInvalidValue;
    fp.d_warps = d_warps;

    auto kern = fused_dispatch_combine_kernel<KMAX, CW, RANKED>;
    int per_sm = 0;
    cudaError_t e = kernel_fit(reinterpret_cast<const void *>(kern), device, threads, smem, &per_sm);
    if (e != cudaSuccess)
        return e;
    if (per_sm < 1)
        return cudaErrorInvalidConfiguration;
    per_sm = std::min(per_sm, tu.fused_ctas_per_sm > 0 ? tu.fused_ctas_per_sm
                              : kWide                     ? kWideCtasPerSm
                                                          : kDefaultCtasPerSm * 4 / CW);

    // work items
    const double d_token_bytes = static_cast<double>(a.d.row_bytes + a.d.srow_bytes) * (1 + a.d.k);
    uint32_t d_run = tu.fused_dispatch_run > 0
                         ? static_cast<uint32_t>(tu.fused_dispatch_run)
                         : static_cast<uint32_t>((a.use_flags ? kDispatchItemBytesFlags
                                                              : kDispatchItemBytes) /
                                                     d_token_bytes +
                                                 0.5);
    d_run = std::min<uint32_t>(std::max<uint32_t>(d_run, 1), 32);  // one flag per lane
    uint32_t c_run = static_cast<uint32_t>(tu.fused_combine_run);
    if (c_run == 0) {
        const double c_token_bytes = static_cast<double>(c.row_bytes) * (1 + a.c.k);
        const double div = a.use_flags && !kWide ? 2.0 : 1.0;
        c_run = static_cast<uint32_t>(kCombineItemBytes / div / c_token_bytes + 0.5);
        c_run = std::min<uint32_t>(std::max<uint32_t>(c_run, 1),
                                   static_cast<uint32_t>(kMaxCombineRun / div));
    }
    fp.d_run_tokens = d_run;
    fp.c_run_tokens = c_run;
    fp.d_items = static_cast<uint32_t>(ceil_div(a.d.N, d_run));
    fp.c_items = static_cast<uint32_t>(ceil_div(a.c.N, c_run));

    // Every CTA the device holds at once, but no more than there are items to take (a
    // small batch would otherwise pay for hundreds of idle CTAs and their counter traffic).
    const int64_t items = ceil_div(fp.d_items, d_warps) + static_cast<int64_t>(fp.c_items);
    const int64_t grid = std::max<int64_t>(
        2, std::min<int64_t>(static_cast<int64_t>(sm_count(device)) * per_sm, items));

    // CTAs that start on dispatch: a share of the grid, at least one when there is
    // dispatch work (the ready flags rely on it) and at least one starting on combine when
    // there is combine work.
    int64_t d_first;
    if (fp.d_items == 0) {
        d_first = 0;
    } else if (fp.c_items == 0) {
        d_first = grid;
    } else {
        const int share = tu.fused_dispatch_share > 0 ? std::min(tu.fused_dispatch_share, 100)
                          : kWide       ? kWideDispatchSharePct
                          : a.use_flags ? kDefaultDispatchSharePctFlags
                                        : kDefaultDispatchSharePct;
        d_first = grid * share / 100;
        d_first = grid < 2 ? grid : std::min<int64_t>(std::max<int64_t>(d_first, 1), grid - 1);
    }
    fp.d_first_ctas = static_cast<uint32_t>(d_first);

    // Only the ready-flag waits need every CTA resident at once (cooperative launch); with
    // no flags no CTA waits on another and an ordinary launch, cheaper to start, is enough.
    return launch_kernel(kern, dim3(static_cast<unsigned>(grid)), dim3(threads), smem, stream,
                         a.use_flags, device, fp);
}

template <bool RANKED>
cudaError_t launch_fused_k(const FusedArgs &a, int device, cudaStream_t stream)
{
    // The combine side takes the separate combine kernel's chunk widths: for k <= 4, eight
    // consumer warps and 4 KB of every row per stage, so that a stage is not a couple of
    // 2 KB rows with a barrier round each.
    const int max_cw = tuning().combine_max_cw > 0 ? tuning().combine_max_cw : 8;
    if (a.c.k <= 4 && max_cw >= 8)
        return launch_fused_shape<4, 8, RANKED>(a, device, stream);
    if (a.c.k <= 8)
        return launch_fused_shape<8, 4, RANKED>(a, device, stream);
    if (a.c.k <= 16)
        return launch_fused_shape<16, 2, RANKED>(a, device, stream);
    return launch_fused_shape<32, 1, RANKED>(a, device, stream);
}

}  // namespace

cudaError_t launch_fused(const FusedArgs &a, int device, cudaStream_t stream)
{
    if (a.d.N == 0 && a.c.N == 0)
        return cudaSuccess;
    return a.c.ranked ? launch_fused_k<true>(a, device, stream)
                      : launch_fused_k<false>(a, device, stream);
}

}  // namespace moe
