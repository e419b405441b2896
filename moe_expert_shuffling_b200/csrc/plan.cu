// Planner: histogram, device-wide prefix scan and stable in-segment rank, plus the
// per-rank dedup lists.  FUSCO (arXiv 2512.22036), abstract: "lightweight planning"
// turns the captured fine-grained layout into placements and removes redundant
// transfers; DySHARP blog, section 5: the destination maps a token's logical index to a
// local address -- slot[t, j] is that map.
//
// Three kernels, all deterministic (counts are order-free; ranks follow token order):
//   plan_count  one CTA per tile of 128 tokens: per-tile expert counts and per-tile
//               counts of (token, rank) moves -> scratch [E][tiles], [R][tiles]
//   plan_scan   one CTA per expert row and per rank row: exclusive scan over tiles,
//               row totals -> cnt[E], rcnt[R]; CTA 0 also gathers the tile flags
//   plan_rank   one CTA per tile: segment starts (scan of cnt/rcnt), entry classes and
//               per-warp counts in parallel over the tile's entries, then each warp
//               walks its 16 tokens in order, one token per step with lane j holding
//               column j.  The valid ids of one token are distinct, so the lanes of a
//               step touch distinct counters and the walk needs no atomics.
#include "common.cuh"
#include "internal.cuh"

namespace moe {
namespace {

constexpr int kPlanThreads = kPlanWarps * 32;
constexpr int kScanThreads = 256;
constexpr uint32_t kFull = 0xffffffffu;  // all lanes of a warp

// Entry classification, shared by the count and rank kernels so both see the same
// entries.  An entry (t, j) is valid when its id is in [0, E) and no earlier column of
// token t holds the same id; a valid entry leads its rank when no earlier valid column
// of t is on the same rank.  Two passes over a tile of ids in shared memory:
//   pass 1: vid[i] = id if valid else -1 (and error flags)
//   pass 2: lead[i] = for a leader, the mask of t's valid columns on its rank, else 0
// Each entry scans only its own token's k <= 32 columns, in parallel over all threads.
__device__ __forceinline__ uint32_t classify_pass1(const int32_t *ids, int32_t *vid, int n_ent,
                                                   int k, int E)
{
    uint32_t flags = 0;
    for (int i = threadIdx.x; i < n_ent; i += blockDim.x) {
        const int j = i % k;
        const int32_t *row = ids + (i - j);
        const int32_t e = row[j];
        bool valid = static_cast<uint32_t>(e) < static_cast<uint32_t>(E);
        if (!valid) {
            flags |= MOE_ERR_ID_RANGE;
        } else {
            for (int q = 0; q < j; ++q)
                if (row[q] == e) {
                    valid = false;
                    flags |= MOE_ERR_ID_DUP;
                    break;
                }
        }
        vid[i] = valid ? e : -1;
    }
    return flags;
}

// Pass 2 for entry i (vid must be complete).  Returns the leader mask (0 if not a leader).
__device__ __forceinline__ uint32_t classify_leader(const int32_t *vid, int i, int k, int epr)
{
    const int j = i % k;
    const int32_t *row = vid + (i - j);
    const int32_t e = row[j];
    if (e < 0)
        return 0u;
    const int32_t r = e / epr;
    uint32_t mask = 0;
    for (int q = 0; q < k; ++q) {
        const int32_t eq = row[q];
        if (eq >= 0 && eq / epr == r) {
            if (q < j)
                return 0u;  // an earlier valid column leads this rank
            mask |= 1u << q;
        }
    }
    return mask;
}

// Exclusive block scan of one value per thread; *total gets the block sum.
// `warp_sums` is shared scratch of blockDim.x / 32 entries.  All threads must call.
__device__ int32_t block_exclusive_scan(int32_t v, int32_t *total, int32_t *warp_sums)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    int32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int32_t y = __shfl_up_sync(kFull, x, o);
        if (lane >= o)
            x += y;
    }
    if (lane == 31)
        warp_sums[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int32_t s = lane < nwarps ? warp_sums[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t y = __shfl_up_sync(kFull, s, o);
            if (lane >= o)
                s += y;
        }
        if (lane < nwarps)
            warp_sums[lane] = s;
    }
    __syncthreads();
    const int32_t before = warp > 0 ? warp_sums[warp - 1] : 0;
    *total = warp_sums[nwarps - 1];
    __syncthreads();
    return before + x - v;
}

// dst[0..n] = exclusive scan of src[0..n) followed by the total.  All threads must call.
__device__ void scan_into(const int32_t *src, int n, int32_t *dst, int32_t *warp_sums)
{
    int32_t carry = 0;
    for (int base = 0; base < n; base += blockDim.x) {
        const int i = base + threadIdx.x;
        const int32_t v = i < n ? src[i] : 0;
        int32_t tot;
        const int32_t ex = block_exclusive_scan(v, &tot, warp_sums);
        if (i < n)
            dst[i] = carry + ex;
        carry += tot;
    }
    if (threadIdx.x == 0)
        dst[n] = carry;
}

__global__ void __launch_bounds__(kPlanThreads)
    plan_count_kernel(const int32_t *__restrict__ topk_idx, int32_t N, int32_t k, int32_t E,
                      int32_t epr, int32_t R, int32_t nt, int32_t *__restrict__ tile_cnt,
                      int32_t *__restrict__ tile_rcnt, uint32_t *__restrict__ tile_err)
{
    extern __shared__ int32_t smem[];
    int32_t *hist = smem;            // [E]
    int32_t *rhist = hist + E;       // [R]
    int32_t *ids = rhist + R;        // [kPlanTile * k]
    int32_t *vid = ids + kPlanTile * k;  // [kPlanTile * k]
    __shared__ uint32_t s_err;

    const int tile = blockIdx.x;
    const int64_t t0 = static_cast<int64_t>(tile) * kPlanTile;
    const int64_t left = N - t0;
    const int ntok = static_cast<int>(left < kPlanTile ? left : kPlanTile);
    const int n_ent = ntok * k;

    for (int i = threadIdx.x; i < E + R; i += blockDim.x)
        smem[i] = 0;
    const int32_t *src = topk_idx + t0 * k;
    for (int i = threadIdx.x; i < n_ent; i += blockDim.x)
        ids[i] = __ldg(src + i);
    if (threadIdx.x == 0)
        s_err = 0;
    __syncthreads();
    const uint32_t flags = classify_pass1(ids, vid, n_ent, k, E);
    if (flags)
        atomicOr(&s_err, flags);
    __syncthreads();
    for (int i = threadIdx.x; i < n_ent; i += blockDim.x) {
        const int32_t e = vid[i];
        if (e < 0)
            continue;
        atomicAdd(&hist[e], 1);
        if (classify_leader(vid, i, k, epr))
            atomicAdd(&rhist[e / epr], 1);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x)
        tile_cnt[static_cast<int64_t>(e) * nt + tile] = hist[e];
    for (int r = threadIdx.x; r < R; r += blockDim.x)
        tile_rcnt[static_cast<int64_t>(r) * nt + tile] = rhist[r];
    if (threadIdx.x == 0)
        tile_err[tile] = s_err;
}

__global__ void __launch_bounds__(kScanThreads)
    plan_scan_kernel(int32_t *__restrict__ tile_cnt, int32_t *__restrict__ tile_rcnt, int32_t E,
                     int32_t R, int32_t nt, int32_t *__restrict__ cnt, int32_t *__restrict__ rcnt,
                     const uint32_t *__restrict__ tile_err, uint32_t *__restrict__ err)
{
    __shared__ int32_t warp_sums[kScanThreads / 32];
    __shared__ uint32_t s_err;
    const int row = blockIdx.x;
    int32_t *p = row < E ? tile_cnt + static_cast<int64_t>(row) * nt
                         : tile_rcnt + static_cast<int64_t>(row - E) * nt;
    int32_t carry = 0;
    for (int base = 0; base < nt; base += blockDim.x) {
        const int i = base + threadIdx.x;
        const int32_t v = i < nt ? p[i] : 0;
        int32_t tot;
        const int32_t ex = block_exclusive_scan(v, &tot, warp_sums);
        if (i < nt)
            p[i] = carry + ex;
        carry += tot;
    }
    if (threadIdx.x == 0) {
        if (row < E)
            cnt[row] = carry;
        else
            rcnt[row - E] = carry;
    }
    if (row == 0) {  // block-uniform
        if (threadIdx.x == 0)
            s_err = 0;
        __syncthreads();
        uint32_t f = 0;
        for (int i = threadIdx.x; i < nt; i += blockDim.x)
            f |= tile_err[i];
        if (f)
            atomicOr(&s_err, f);
        __syncthreads();
        if (threadIdx.x == 0)
            *err = s_err;
    }
}

__global__ void __launch_bounds__(kPlanThreads)
    plan_rank_kernel(const int32_t *__restrict__ topk_idx, int32_t N, int32_t k, int32_t E,
                     int32_t epr, int32_t R, int32_t nt, const int32_t *__restrict__ tile_cnt,
                     const int32_t *__restrict__ tile_rcnt, const int32_t *__restrict__ cnt,
                     const int32_t *__restrict__ rcnt, int32_t *__restrict__ expert_off,
                     int32_t *__restrict__ rank_off, int32_t *__restrict__ rtok_off,
                     int32_t *__restrict__ slot, int32_t *__restrict__ src_tok,
                     int32_t *__restrict__ src_j, int32_t *__restrict__ rtok,
                     uint32_t *__restrict__ fanout, int32_t n_rows, int64_t rtok_cap,
                     uint32_t *__restrict__ err)
{
    extern __shared__ int32_t smem[];
    int32_t *eoff = smem;                       // [E+1]
    int32_t *roff = eoff + E + 1;               // [R+1]
    int32_t *wcnt = roff + R + 1;               // [warps][E]
    int32_t *wrcnt = wcnt + kPlanWarps * E;     // [warps][R]
    int32_t *ids = wrcnt + kPlanWarps * R;      // [kPlanTile * k]
    int32_t *vid = ids + kPlanTile * k;         // [kPlanTile * k]
    uint32_t *lead = reinterpret_cast<uint32_t *>(vid + kPlanTile * k);  // [kPlanTile * k]
    __shared__ int32_t warp_sums[kPlanThreads / 32];

    const int tile = blockIdx.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t t0 = static_cast<int64_t>(tile) * kPlanTile;
    const int64_t left = N - t0;
    const int ntok = static_cast<int>(left <= 0 ? 0 : (left < kPlanTile ? left : kPlanTile));
    const int n_ent = ntok * k;

    // Segment starts: exclusive scans of the expert and rank totals.
    scan_into(cnt, E, eoff, warp_sums);
    scan_into(rcnt, R, roff, warp_sums);
    for (int i = threadIdx.x; i < kPlanWarps * (E + R); i += blockDim.x)
        wcnt[i] = 0;  // wcnt and wrcnt are contiguous
    const int32_t *src = topk_idx + t0 * k;
    for (int i = threadIdx.x; i < n_ent; i += blockDim.x)
        ids[i] = __ldg(src + i);
    __syncthreads();
    if (tile == 0) {
        for (int i = threadIdx.x; i <= E; i += blockDim.x)
            expert_off[i] = eoff[i];
        for (int i = threadIdx.x; i <= R; i += blockDim.x) {
            rtok_off[i] = roff[i];
            rank_off[i] = eoff[i * epr];
        }
    }
    if (ntok == 0)
        return;  // block-uniform; no barrier follows for this block

    classify_pass1(ids, vid, n_ent, k, E);  // flags were reported by the count kernel
    __syncthreads();
    // Leader masks and per-warp counts (warp w owns tokens [16w, 16w + 16) of the tile).
    for (int i = threadIdx.x; i < n_ent; i += blockDim.x) {
        const int32_t e = vid[i];
        uint32_t m = 0;
        if (e >= 0) {
            const int w = (i / k) / kPlanTokensPerWarp;
            atomicAdd(&wcnt[w * E + e], 1);
            m = classify_leader(vid, i, k, epr);
            if (m)
                atomicAdd(&wrcnt[w * R + e / epr], 1);
        }
        lead[i] = m;
    }
    __syncthreads();

    // Start of each warp's run: segment start + earlier tiles + earlier warps of this tile.
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int32_t run = eoff[e] + tile_cnt[static_cast<int64_t>(e) * nt + tile];
        for (int w = 0; w < kPlanWarps; ++w) {
            const int32_t v = wcnt[w * E + e];
            wcnt[w * E + e] = run;
            run += v;
        }
    }
    for (int r = threadIdx.x; r < R; r += blockDim.x) {
        int32_t run = roff[r] + tile_rcnt[static_cast<int64_t>(r) * nt + tile];
        for (int w = 0; w < kPlanWarps; ++w) {
            const int32_t v = wrcnt[w * R + r];
            wrcnt[w * R + r] = run;
            run += v;
        }
    }
    __syncthreads();

    // Ordered walk: one token per step, lane j = column j.  The valid columns of a token
    // hold distinct experts and its leaders distinct ranks, so the lanes of one step never
    // touch the same counter.
    int32_t *my_cnt = wcnt + warp * E;
    int32_t *my_rcnt = wrcnt + warp * R;
    const int tw0 = warp * kPlanTokensPerWarp;
    uint32_t flags = 0;
    for (int q = 0; q < kPlanTokensPerWarp; ++q) {
        const int tl = tw0 + q;
        if (tl >= ntok)
            break;  // warp-uniform
        const int64_t t = t0 + tl;
        if (lane < k) {
            const int i = tl * k + lane;
            const int32_t e = vid[i];
            int32_t s = -1;
            if (e >= 0) {
                s = my_cnt[e];
                my_cnt[e] = s + 1;
                if (static_cast<uint32_t>(s) < static_cast<uint32_t>(n_rows)) {
                    src_tok[s] = static_cast<int32_t>(t);
                    src_j[s] = lane;
                } else {
                    flags |= MOE_ERR_BOUNDS;
                    s = -1;
                }
                const uint32_t m = lead[i];
                if (m) {
                    const int32_t r = e / epr;
                    const int32_t pos = my_rcnt[r];
                    my_rcnt[r] = pos + 1;
                    if (pos >= 0 && pos < rtok_cap) {
                        rtok[pos] = static_cast<int32_t>(t);
                        fanout[pos] = m;
                    } else {
                        flags |= MOE_ERR_BOUNDS;
                    }
                }
            }
            slot[t * k + lane] = s;
        }
        __syncwarp();
    }
    if (flags)
        atomicOr(err, flags);
}

size_t count_smem(int E, int R, int k) { return sizeof(int32_t) * (E + R + 2 * kPlanTile * k); }
size_t rank_smem(int E, int R, int k)
{
    return sizeof(int32_t) *
           ((E + 1) + (R + 1) + static_cast<size_t>(kPlanWarps) * (E + R) + 3 * kPlanTile * k);
}

}  // namespace

cudaError_t launch_plan(moe_plan_s *p, const int32_t *topk_idx, cudaStream_t stream)
{
    static bool attrs_set[64] = {false};
    const int dev = p->device >= 0 && p->device < 64 ? p->device : 0;
    if (!attrs_set[dev]) {
        const int max_rank = static_cast<int>(rank_smem(kMaxExperts, kMaxExperts, kMaxTopk));
        const int max_count = static_cast<int>(count_smem(kMaxExperts, kMaxExperts, kMaxTopk));
        cudaError_t e1 = cudaFuncSetAttribute(plan_rank_kernel,
                                              cudaFuncAttributeMaxDynamicSharedMemorySize, max_rank);
        if (e1 != cudaSuccess)
            return e1;
        e1 = cudaFuncSetAttribute(plan_count_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  max_count);
        if (e1 != cudaSuccess)
            return e1;
        attrs_set[dev] = true;
    }
    const int32_t N = p->N, k = p->k, E = p->E, R = p->R, epr = p->epr;
    const int32_t nt = static_cast<int32_t>(ceil_div(N, kPlanTile));
    const int32_t n_rows = N * k;
    if (nt > 0) {
        plan_count_kernel<<<nt, kPlanThreads, count_smem(E, R, k), stream>>>(
            topk_idx, N, k, E, epr, R, nt, p->tile_cnt, p->tile_rcnt, p->tile_err);
    }
    plan_scan_kernel<<<E + R, kScanThreads, 0, stream>>>(p->tile_cnt, p->tile_rcnt, E, R, nt,
                                                          p->cnt, p->rcnt, p->tile_err, p->err);
    plan_rank_kernel<<<nt > 0 ? nt : 1, kPlanThreads, rank_smem(E, R, k), stream>>>(
        topk_idx, N, k, E, epr, R, nt, p->tile_cnt, p->tile_rcnt, p->cnt, p->rcnt, p->expert_off,
        p->rank_off, p->rtok_off, p->slot, p->src_tok, p->src_j, p->rtok, p->fanout, n_rows,
        p->rtok_cap, p->err);
    return cudaGetLastError();
}

}  // namespace moe
