// Planner: histogram, device-wide prefix scan and stable in-segment rank, plus the
// per-rank dedup lists.  FUSCO (arXiv 2512.22036), abstract: "lightweight planning"
// turns the captured fine-grained layout into placements and removes redundant
// transfers; DySHARP blog, section 5: the destination maps a token's logical index to a
// local address -- slot[t, j] is that map.
//
// Three phases, all deterministic (no result depends on thread timing):
//   count  per tile of 128 tokens: classify the entries, mark each token in 128-bit
//          per-expert and per-rank tile masks; the counts are their popcounts
//          -> scratch [E][tiles], [R][tiles], plus the tile's error flags
//   scan   per expert row and per rank row: exclusive scan over tiles, row totals
//          -> cnt[E], rcnt[R]; the tile flags are gathered into the error word
//   rank   per tile: segment starts, then every entry's stable rank inside its segment
//          as a popcount over a per-expert bitmask of the tile's tokens (bit t set when
//          token t selects the expert), so no step is sequential.
// By default the phases run in one cooperative kernel (plan_fused_kernel) whose CTAs
// meet at two sense-reversing grid barriers; a wait gives up after 1 s and reports
// MOE_ERR_TIMEOUT.  A routing of at most one tile (N <= 128, e.g. a decode step) runs
// all phases in one CTA (plan_one_tile_kernel).  Larger routings run on thread-block
// clusters of up to 16 tiles whose counts are combined through distributed shared memory,
// with one grid-wide exchange of the groups' totals when there is more than one group
// (plan_group_kernel); the cooperative kernel is the fallback when those clusters cannot
// all be resident, and three kernels when its grid cannot be co-resident either.
//
// Inside a tile a warp looks at several tokens at once: lane = (token, column) with the
// columns of one token in a segment of W = next power of two >= k lanes, so a token's
// k ids are compared with width-W shuffles.
#include <algorithm>

#include <cooperative_groups.h>

#include "common.cuh"
#include "internal.cuh"

namespace moe {
namespace {

constexpr int kPlanThreads = kPlanWarps * 32;
constexpr int kScanThreads = 256;
constexpr uint32_t kFull = 0xffffffffu;  // all lanes of a warp

// Kernel parameters: shape, routing, outputs and scratch.
struct PlanK {
    const int32_t *topk_idx;
    int32_t N, k, E, R, epr, nt, n_rows, align;
    int32_t match;  // classify with warp match instructions (1) or shuffle compares (0)
    int32_t lists;  // write the per-rank dedup lists rtok / fanout (0: skip them)
    int64_t rtok_cap;
    int32_t *tile_cnt, *tile_rcnt;
    uint32_t *tile_err;
    int32_t *cnt, *expert_off, *rcnt, *rank_off, *rtok_off, *slot, *src_tok, *src_j, *rtok;
    uint32_t *fanout, *err;
    uint32_t *sync;  // [2] grid-barrier arrival count (zero at rest) and generation
    uint32_t *group_flag;  // [groups] arrival words of the group kernel
};

// Classification of one entry, shared by the count and rank kernels so both see the
// same entries.  Entry (t, j) is valid when its id is in [0, E) and no earlier column of
// token t holds the same id; a valid entry leads its rank when no earlier valid column
// of t is on that rank, and then carries the mask of t's valid columns on the rank.
struct Entry {
    int32_t e;        // the id if valid, else -1
    int32_t r;        // its rank if valid, else -1
    uint32_t lead;    // mask of the token's valid columns on rank r if this entry leads
    uint32_t flags;   // MOE_ERR_* raised by this entry
};

// Lane layout of a warp step: `wbits` = log2 of the segment width W >= k.
struct LaneMap {
    int wbits, per_step, steps;
};

__device__ __forceinline__ LaneMap lane_map(int k)
{
    LaneMap m;
    m.wbits = 0;
    while ((1 << m.wbits) < k)
        ++m.wbits;
    m.per_step = 32 >> m.wbits;  // tokens per warp step
    m.steps = (kPlanTokensPerWarp + m.per_step - 1) / m.per_step;
    return m;
}

// All 32 lanes must call.  `tl` is the token's index in the tile, `present` whether
// this lane holds an entry (token in range and column < k); W >= k is the width of a token's
// lane segment.  The W shuffles of each comparison are independent of one another (the
// loops are unrolled), so they issue back to back instead of one round trip each; lanes
// q >= k of a segment hold id -1 and rank -1, which match no valid entry.
template <int W>
__device__ __forceinline__ Entry classify(const int32_t *ids, const int32_t *rank_of, int tl,
                                          int j, bool present, int k, int E)
{
    Entry c;
    const int32_t id = present ? ids[tl * k + j] : -1;
    const bool in_range = present && static_cast<uint32_t>(id) < static_cast<uint32_t>(E);
    int32_t other[W];
#pragma unroll
    for (int q = 0; q < W; ++q)
        other[q] = __shfl_sync(kFull, id, q, W);
    bool valid = in_range;
#pragma unroll
    for (int q = 0; q < W; ++q)
        if (q < j && other[q] == id)
            valid = false;
    // -1 marks an entry the router dropped: no row, no contribution, not an error
    c.flags = (present && !in_range && id != -1 ? MOE_ERR_ID_RANGE : 0u) |
              (in_range && !valid ? MOE_ERR_ID_DUP : 0u);
    c.e = valid ? id : -1;
    c.r = valid ? rank_of[id] : -1;
#pragma unroll
    for (int q = 0; q < W; ++q)
        other[q] = __shfl_sync(kFull, c.r, q, W);
    uint32_t mask = 0;
    bool leader = valid;
#pragma unroll
    for (int q = 0; q < W; ++q) {
        if (valid && other[q] == c.r) {
            if (q < j)
                leader = false;
            mask |= 1u << q;
        }
    }
    c.lead = leader ? mask : 0u;
    return c;
}

// Number of set bits of a 128-bit tile mask below bit `tl`.
__device__ __forceinline__ int32_t bits_below(const uint32_t *m4, int tl)
{
    const int w = tl >> 5;
    int32_t n = __popc(m4[w] & ((1u << (tl & 31)) - 1u));
    for (int q = 0; q < w; ++q)
        n += __popc(m4[q]);
    return n;
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

// dst[0..n] = exclusive scan of src[0..n) followed by the total, by one warp (n <= 1024):
// each lane sums a run of consecutive values, a warp scan offsets the runs.  No block
// barrier is taken, so two warps can scan two arrays at once.
__device__ void warp_scan_into(const int32_t *src, int n, int32_t *dst)
{
    const int lane = threadIdx.x & 31;
    const int per = (n + 31) / 32;
    const int b = lane * per;
    int32_t sum = 0;
    for (int i = 0; i < per; ++i)
        if (b + i < n)
            sum += src[b + i];
    int32_t incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int32_t y = __shfl_up_sync(kFull, incl, o);
        if (lane >= o)
            incl += y;
    }
    int32_t run = incl - sum;
    for (int i = 0; i < per; ++i)
        if (b + i < n) {
            const int32_t v = src[b + i];
            dst[b + i] = run;
            run += v;
        }
    if (lane == 31)
        dst[n] = incl;
}

// Shared-memory layout of every plan kernel (words).  The ids come first so that they are
// 16-byte aligned for vector loads (kPlanTile * k words is a multiple of 4).
struct PlanSmem {
    int32_t *ids;       // [kPlanTile * k] the tile's routing ids
    int32_t *vid;       // [kPlanTile * k] valid id or -1
    uint32_t *lead;     // [kPlanTile * k] leader masks
    int32_t *eoff;      // [E+1] segment starts of the experts
    int32_t *roff;      // [R+1] starts of the ranks' dedup lists
    int32_t *ebase;     // [E]   tile base per expert; the histogram while counting
    int32_t *rbase;     // [R]   tile base per rank; the rank histogram while counting
    int32_t *rank_of;   // [E]   rank of each expert
    uint32_t *emask;    // [E][4] tokens of the tile on each expert
    uint32_t *rmask;    // [R][4] tokens of the tile on each rank
    int32_t *end;       // first word after the layout
};

__host__ __device__ constexpr size_t plan_smem_words(int E, int R, int k)
{
    return static_cast<size_t>(E + 1) + (R + 1) + E + R + E + 4 * E + 4 * R +
           3 * static_cast<size_t>(kPlanTile) * k;
}

__device__ PlanSmem carve(int32_t *w, int E, int R, int k)
{
    PlanSmem m;
    m.ids = w;
    m.vid = m.ids + kPlanTile * k;
    m.lead = reinterpret_cast<uint32_t *>(m.vid + kPlanTile * k);
    m.eoff = reinterpret_cast<int32_t *>(m.lead + kPlanTile * k);
    m.roff = m.eoff + E + 1;
    m.ebase = m.roff + R + 1;
    m.rbase = m.ebase + E;
    m.rank_of = m.rbase + R;
    m.emask = reinterpret_cast<uint32_t *>(m.rank_of + E);
    m.rmask = m.emask + 4 * E;
    m.end = reinterpret_cast<int32_t *>(m.rmask + 4 * R);
    return m;
}

__device__ __forceinline__ int tile_tokens(const PlanK &p, int tile)
{
    const int64_t left = static_cast<int64_t>(p.N) - static_cast<int64_t>(tile) * kPlanTile;
    return static_cast<int>(left <= 0 ? 0 : (left < kPlanTile ? left : kPlanTile));
}

__device__ void init_rank_of(const PlanK &p, const PlanSmem &m)
{
    for (int e = threadIdx.x; e < p.E; e += blockDim.x)
        m.rank_of[e] = e / p.epr;
}

// The tile's ids into shared memory in one round trip: every thread issues all of its
// loads (16-byte vectors when the tile's ids are 16-byte aligned) before storing any.
__device__ void load_ids(const PlanK &p, const PlanSmem &m, int tile, int ntok)
{
    constexpr int kVecPerThread = kPlanTile * kMaxTopk / 4 / kPlanThreads;  // 4
    const int32_t *src = p.topk_idx + static_cast<int64_t>(tile) * kPlanTile * p.k;
    const int n = ntok * p.k;
    int head = 0;
    if ((reinterpret_cast<uintptr_t>(src) & 15u) == 0 && (smem_addr(m.ids) & 15u) == 0) {
        const int n4 = n >> 2;
        const int4 *s4 = reinterpret_cast<const int4 *>(src);
        int4 v[kVecPerThread];
#pragma unroll
        for (int q = 0; q < kVecPerThread; ++q) {
            const int i = threadIdx.x + q * kPlanThreads;
            if (i < n4)
                v[q] = __ldg(s4 + i);
        }
#pragma unroll
        for (int q = 0; q < kVecPerThread; ++q) {
            const int i = threadIdx.x + q * kPlanThreads;
            if (i < n4)
                reinterpret_cast<int4 *>(m.ids)[i] = v[q];
        }
        head = 4 * n4;
    }
    constexpr int kPerThread = 4;
    for (int base = head; base < n; base += kPerThread * kPlanThreads) {
        int32_t v[kPerThread];
#pragma unroll
        for (int q = 0; q < kPerThread; ++q) {
            const int i = base + threadIdx.x + q * kPlanThreads;
            if (i < n)
                v[q] = __ldg(src + i);
        }
#pragma unroll
        for (int q = 0; q < kPerThread; ++q) {
            const int i = base + threadIdx.x + q * kPlanThreads;
            if (i < n)
                m.ids[i] = v[q];
        }
    }
}

__device__ __forceinline__ void clear_tile_masks(const PlanK &p, const PlanSmem &m)
{
    for (int i = threadIdx.x; i < 4 * (p.E + p.R); i += blockDim.x)
        m.emask[i] = 0u;  // emask and rmask are contiguous
}

__device__ uint32_t classify_loaded(const PlanK &p, const PlanSmem &m, int ntok);

// Classify a tile's entries into shared memory: vid/lead per entry, and each token's bit
// in its experts' and ranks' tile masks.  All threads must call; rank_of must be ready.
// Returns this thread's MOE_ERR_* flags.
__device__ uint32_t classify_tile(const PlanK &p, const PlanSmem &m, int tile, int ntok)
{
    clear_tile_masks(p, m);
    load_ids(p, m, tile, ntok);
    return classify_loaded(p, m, ntok);
}

// classify<W> with two warp match instructions instead of 2W shuffle compares: lanes whose
// (token, id) keys match hold the same expert, and the lowest of them is the first column;
// lanes whose (token, rank) keys match are the token's valid columns on one rank.  Lanes
// without a valid key get one no other lane has.  Ids are below 2^20 (E <= 1024), token
// segments below 32.
template <int W>
__device__ __forceinline__ Entry classify_match(const int32_t *ids, const int32_t *rank_of,
                                                int tl, int j, bool present, int k, int E)
{
    Entry c;
    const int lane = threadIdx.x & 31;
    const uint32_t seg = static_cast<uint32_t>(lane / W);
    const int32_t id = present ? ids[tl * k + j] : -1;
    const bool in_range = present && static_cast<uint32_t>(id) < static_cast<uint32_t>(E);
    const uint32_t key = in_range ? (seg << 20) | static_cast<uint32_t>(id)
                                  : 0x80000000u | static_cast<uint32_t>(lane);
    const uint32_t same = __match_any_sync(kFull, key);
    const bool valid = in_range && __ffs(same) - 1 == lane;
    c.flags = (present && !in_range && id != -1 ? MOE_ERR_ID_RANGE : 0u) |
              (in_range && !valid ? MOE_ERR_ID_DUP : 0u);
    c.e = valid ? id : -1;
    c.r = valid ? rank_of[id] : -1;
    const uint32_t rkey = valid ? (seg << 20) | static_cast<uint32_t>(c.r)
                                : 0x80000000u | static_cast<uint32_t>(lane);
    const uint32_t rsame = __match_any_sync(kFull, rkey);
    const bool leader = valid && __ffs(rsame) - 1 == lane;
    const uint32_t cols = W == 32 ? 0xffffffffu : (1u << W) - 1u;
    c.lead = leader ? (rsame >> (seg * W)) & cols : 0u;
    return c;
}

// The warp steps of classify_loaded for one lane-segment width W (a power of two >= k).
template <int W>
__device__ __forceinline__ uint32_t classify_steps(const PlanK &p, const PlanSmem &m, int ntok)
{
    constexpr int kWbits = W == 1 ? 0 : W == 2 ? 1 : W == 4 ? 2 : W == 8 ? 3 : W == 16 ? 4 : 5;
    constexpr int kPerStep = 32 / W;  // tokens per warp step
    constexpr int kSteps = (kPlanTokensPerWarp + kPerStep - 1) / kPerStep;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int k = p.k;
    const int j = lane & (W - 1);
    const int sub = lane >> kWbits;
    uint32_t flags = 0;
#pragma unroll 1
    for (int st = 0; st < kSteps; ++st) {
        const int tw = st * kPerStep + sub;           // token within the warp's 16
        const int tl = warp * kPlanTokensPerWarp + tw;
        const bool present = tw < kPlanTokensPerWarp && tl < ntok && j < k;
        const Entry c = p.match ? classify_match<W>(m.ids, m.rank_of, tl, j, present, k, p.E)
                                : classify<W>(m.ids, m.rank_of, tl, j, present, k, p.E);
        flags |= c.flags;
        if (present) {
            m.vid[tl * k + j] = c.e;
            m.lead[tl * k + j] = c.lead;
            const uint32_t bit = 1u << (tl & 31);
            if (c.e >= 0)
                atomicOr(&m.emask[4 * c.e + (tl >> 5)], bit);
            if (c.lead)
                atomicOr(&m.rmask[4 * c.r + (tl >> 5)], bit);
        }
    }
    return flags;
}

// classify_loaded for the lane-segment widths up to WMAX only (kernels instantiated per range
// of k carry only the widths they need).
template <int WMAX>
__device__ uint32_t classify_loaded_w(const PlanK &p, const PlanSmem &m, int ntok)
{
    __syncthreads();
    uint32_t flags;
    const int w = 1 << lane_map(p.k).wbits;  // block-uniform
    if (WMAX > 16 && w > 16)
        flags = classify_steps<32>(p, m, ntok);
    else if (w > 8)
        flags = classify_steps<16>(p, m, ntok);
    else if (w > 4)
        flags = classify_steps<8>(p, m, ntok);
    else if (w > 2)
        flags = classify_steps<4>(p, m, ntok);
    else if (w > 1)
        flags = classify_steps<2>(p, m, ntok);
    else
        flags = classify_steps<1>(p, m, ntok);
    __syncthreads();
    return flags;
}

// classify_tile once the masks are clear and the ids are being stored (synchronises first).
__device__ uint32_t classify_loaded(const PlanK &p, const PlanSmem &m, int ntok)
{
    __syncthreads();
    uint32_t flags;
    switch (1 << lane_map(p.k).wbits) {  // block-uniform
    case 1: flags = classify_steps<1>(p, m, ntok); break;
    case 2: flags = classify_steps<2>(p, m, ntok); break;
    case 4: flags = classify_steps<4>(p, m, ntok); break;
    case 8: flags = classify_steps<8>(p, m, ntok); break;
    case 16: flags = classify_steps<16>(p, m, ntok); break;
    default: flags = classify_steps<32>(p, m, ntok); break;
    }
    __syncthreads();
    return flags;
}

// Count phase for one tile: the tile's count per expert (per rank) is the number of its
// tokens on it, the popcount of the tile mask.  Leaves the tile's classification in
// shared memory.  All threads must call; rank_of must be ready.
__device__ void count_tile(const PlanK &p, const PlanSmem &m, int tile, uint32_t *s_err)
{
    if (threadIdx.x == 0)
        *s_err = 0;
    const uint32_t flags = classify_tile(p, m, tile, tile_tokens(p, tile));
    if (flags)
        atomicOr(s_err, flags);
    for (int e = threadIdx.x; e < p.E; e += blockDim.x) {
        const uint32_t *mk = &m.emask[4 * e];
        p.tile_cnt[static_cast<int64_t>(e) * p.nt + tile] =
            __popc(mk[0]) + __popc(mk[1]) + __popc(mk[2]) + __popc(mk[3]);
    }
    for (int r = threadIdx.x; r < p.R; r += blockDim.x) {
        const uint32_t *mk = &m.rmask[4 * r];
        p.tile_rcnt[static_cast<int64_t>(r) * p.nt + tile] =
            __popc(mk[0]) + __popc(mk[1]) + __popc(mk[2]) + __popc(mk[3]);
    }
    __syncthreads();
    if (threadIdx.x == 0)
        p.tile_err[tile] = *s_err;
    __syncthreads();
}

// Segment offsets from m.ebase (segment sizes: the counts rounded up to the alignment) and
// m.rbase (rank counts), which the caller has filled; `raw_cnt` holds the expert counts
// (shared memory when `raw_shared`, else the global cnt array).  Block 0 writes the offset
// arrays; every receive row that no entry maps to (segment padding and rows after the last
// segment) is marked -1 in src_tok/src_j, spread over all CTAs of the grid.
__device__ void prepare_offsets(const PlanK &p, const PlanSmem &m, const int32_t *raw_cnt,
                                bool raw_shared);

__device__ void rank_prepare(const PlanK &p, const PlanSmem &m)
{
    for (int i = threadIdx.x; i < p.E + p.R; i += blockDim.x) {
        if (i < p.E) {
            const int32_t c = __ldcg(p.cnt + i);
            m.ebase[i] = (c + p.align - 1) / p.align * p.align;
        } else {
            m.rbase[i - p.E] = __ldcg(p.rcnt + (i - p.E));
        }
    }
    prepare_offsets(p, m, p.cnt, false);
}

__device__ void prepare_offsets(const PlanK &p, const PlanSmem &m, const int32_t *raw_cnt,
                                bool raw_shared)
{
    __syncthreads();
    if (threadIdx.x < 32)
        warp_scan_into(m.ebase, p.E, m.eoff);
    else if (threadIdx.x < 64)
        warp_scan_into(m.rbase, p.R, m.roff);
    __syncthreads();
    if (blockIdx.x == 0) {
        for (int i = threadIdx.x; i <= p.E; i += blockDim.x)
            p.expert_off[i] = m.eoff[i];
        for (int i = threadIdx.x; i <= p.R; i += blockDim.x) {
            p.rtok_off[i] = m.roff[i];
            p.rank_off[i] = m.eoff[i * p.epr];
        }
    }
    if (p.align > 1) {
        for (int e = blockIdx.x; e < p.E; e += gridDim.x) {
            const int32_t first = m.eoff[e] + (raw_shared ? raw_cnt[e] : __ldcg(raw_cnt + e));
            for (int32_t r = first + threadIdx.x; r < m.eoff[e + 1]; r += blockDim.x) {
                p.src_tok[r] = -1;
                p.src_j[r] = -1;
            }
        }
    }
    for (int64_t r = m.eoff[p.E] + static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
         r < p.n_rows; r += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        p.src_tok[r] = -1;
        p.src_j[r] = -1;
    }
}

__device__ void rank_entries(const PlanK &p, const PlanSmem &m, int tile, int ntok);

// Rank phase for one tile.  All threads must call; rank_prepare must have run.  With
// tile_ready the tile's classification (count_tile of this tile) is still in shared
// memory; otherwise it is rebuilt.
__device__ void rank_tile(const PlanK &p, const PlanSmem &m, int tile, bool tile_ready)
{
    const int ntok = tile_tokens(p, tile);
    if (ntok == 0)
        return;  // block-uniform
    if (!tile_ready)
        (void)classify_tile(p, m, tile, ntok);  // flags were reported by the count phase
    // This tile's first receive row per expert and first dedup entry per rank.
    for (int e = threadIdx.x; e < p.E; e += blockDim.x)
        m.ebase[e] = m.eoff[e] + __ldcg(p.tile_cnt + static_cast<int64_t>(e) * p.nt + tile);
    for (int r = threadIdx.x; r < p.R; r += blockDim.x)
        m.rbase[r] = m.roff[r] + __ldcg(p.tile_rcnt + static_cast<int64_t>(r) * p.nt + tile);
    __syncthreads();
    rank_entries(p, m, tile, ntok);
}

// Stable rank of every entry of a classified tile whose bases m.ebase / m.rbase are set:
// tile base + earlier tokens of the tile on the same expert.  All threads must call.
__device__ void rank_entries(const PlanK &p, const PlanSmem &m, int tile, int ntok)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int k = p.k;
    const LaneMap lm = lane_map(k);
    const int j = lane & ((1 << lm.wbits) - 1);
    const int sub = lane >> lm.wbits;
    const int64_t t0 = static_cast<int64_t>(tile) * kPlanTile;
    uint32_t flags = 0;
    for (int st = 0; st < lm.steps; ++st) {
        const int tw = st * lm.per_step + sub;
        const int tl = warp * kPlanTokensPerWarp + tw;
        if (!(tw < kPlanTokensPerWarp && tl < ntok && j < k))
            continue;
        const int64_t t = t0 + tl;
        const int i = tl * k + j;
        const int32_t e = m.vid[i];
        int32_t s = -1;
        if (e >= 0) {
            s = m.ebase[e] + bits_below(&m.emask[4 * e], tl);
            if (static_cast<uint32_t>(s) < static_cast<uint32_t>(p.n_rows)) {
                p.src_tok[s] = static_cast<int32_t>(t);
                p.src_j[s] = j;
            } else {
                flags |= MOE_ERR_BOUNDS;
                s = -1;
            }
            const uint32_t msk = m.lead[i];
            if (msk && p.lists) {
                const int32_t r = m.rank_of[e];
                const int32_t pos = m.rbase[r] + bits_below(&m.rmask[4 * r], tl);
                if (pos >= 0 && pos < p.rtok_cap) {
                    p.rtok[pos] = static_cast<int32_t>(t);
                    p.fanout[pos] = msk;
                } else {
                    flags |= MOE_ERR_BOUNDS;
                }
            }
        }
        p.slot[t * k + j] = s;
    }
    if (flags)
        atomicOr(p.err, flags);
    __syncthreads();
}

// ------------------------------------------------------------- three-kernel path
__global__ void __launch_bounds__(kPlanThreads) plan_count_kernel(const PlanK p)
{
    extern __shared__ __align__(16) int32_t smem[];
    __shared__ uint32_t s_err;
    const PlanSmem m = carve(smem, p.E, p.R, p.k);
    init_rank_of(p, m);
    pdl_wait();
    count_tile(p, m, blockIdx.x, &s_err);
    pdl_trigger();  // late, so that the next kernel's CTAs do not wait beside this one's work
}

__global__ void __launch_bounds__(kScanThreads) plan_scan_kernel(const PlanK p)
{
    __shared__ int32_t warp_sums[kScanThreads / 32];
    __shared__ uint32_t s_err;
    pdl_wait();
    const int row = blockIdx.x;
    int32_t *rp = row < p.E ? p.tile_cnt + static_cast<int64_t>(row) * p.nt
                            : p.tile_rcnt + static_cast<int64_t>(row - p.E) * p.nt;
    int32_t carry = 0;
    for (int base = 0; base < p.nt; base += blockDim.x) {
        const int i = base + threadIdx.x;
        const int32_t v = i < p.nt ? rp[i] : 0;
        int32_t tot;
        const int32_t ex = block_exclusive_scan(v, &tot, warp_sums);
        if (i < p.nt)
            rp[i] = carry + ex;
        carry += tot;
    }
    if (threadIdx.x == 0) {
        if (row < p.E)
            p.cnt[row] = carry;
        else
            p.rcnt[row - p.E] = carry;
    }
    if (row == 0) {  // block-uniform
        if (threadIdx.x == 0)
            s_err = 0;
        __syncthreads();
        uint32_t f = 0;
        for (int i = threadIdx.x; i < p.nt; i += blockDim.x)
            f |= p.tile_err[i];
        if (f)
            atomicOr(&s_err, f);
        __syncthreads();
        if (threadIdx.x == 0)
            *p.err = s_err;
    }
    pdl_trigger();
}

__global__ void __launch_bounds__(kPlanThreads) plan_rank_kernel(const PlanK p)
{
    extern __shared__ __align__(16) int32_t smem[];
    const PlanSmem m = carve(smem, p.E, p.R, p.k);
    init_rank_of(p, m);
    pdl_wait();
    rank_prepare(p, m);
    pdl_trigger();
    rank_tile(p, m, blockIdx.x, false);
}

// ------------------------------------------------------------- one tile (N <= 128)
// Every phase in one CTA: the counts are the popcounts of the single tile's masks, so no
// scratch, no grid barrier and no cooperative launch is needed.
__global__ void __launch_bounds__(kPlanThreads) plan_one_tile_kernel(const PlanK p)
{
    extern __shared__ __align__(16) int32_t smem[];
    __shared__ uint32_t s_err;
    const PlanSmem m = carve(smem, p.E, p.R, p.k);
    if (threadIdx.x == 0)
        s_err = 0;
    pdl_trigger();
    init_rank_of(p, m);
    pdl_wait();  // the routing and the plan's arrays are accessed from here on
    const int ntok = tile_tokens(p, 0);
    const uint32_t flags = classify_tile(p, m, 0, ntok);  // synchronises first
    if (flags)
        atomicOr(&s_err, flags);
    for (int e = threadIdx.x; e < p.E; e += blockDim.x) {
        const uint32_t *mk = &m.emask[4 * e];
        const int32_t c = __popc(mk[0]) + __popc(mk[1]) + __popc(mk[2]) + __popc(mk[3]);
        p.cnt[e] = c;
        m.ebase[e] = (c + p.align - 1) / p.align * p.align;
    }
    for (int r = threadIdx.x; r < p.R; r += blockDim.x) {
        const uint32_t *mk = &m.rmask[4 * r];
        const int32_t c = __popc(mk[0]) + __popc(mk[1]) + __popc(mk[2]) + __popc(mk[3]);
        p.rcnt[r] = c;
        m.rbase[r] = c;
    }
    __syncthreads();
    if (threadIdx.x == 0)
        *p.err = s_err;  // before any MOE_ERR_BOUNDS of the rank step is or-ed in
    prepare_offsets(p, m, p.cnt, false);
    // the tile's bases are the segment starts themselves
    for (int e = threadIdx.x; e < p.E; e += blockDim.x)
        m.ebase[e] = m.eoff[e];
    for (int r = threadIdx.x; r < p.R; r += blockDim.x)
        m.rbase[r] = m.roff[r];
    __syncthreads();
    if (ntok > 0)  // block-uniform
        rank_entries(p, m, 0, ntok);
}

// ------------------------------------------- groups of tiles on thread-block clusters
// One CTA per tile; the CTAs are grouped C at a time (C <= 16) into thread-block clusters.
//  1. Each CTA counts its tile, stores the counts column-wise (row * tiles + tile) and
//     releases its arrival word.  (A grid of one cluster skips the global exchange: after a
//     cluster barrier its CTAs read the counts straight from each other's shared memory.)
//  2. While the other tiles arrive, it prepares everything that depends only on its own
//     tile: the tile-local offset of every expert and rank (scans of the tile counts) and a
//     staging order of the tile's entries by (expert, token) and of its leaders by (rank,
//     token) in shared memory.
//  3. Once every CTA has arrived, each CTA of a cluster scans its share of the rows (1/C of
//     them) across all tiles with coalesced loads, and writes through distributed shared
//     memory, into each CTA of its cluster, that tile's prefix of the row (its base) and
//     the row's total.
//  4. After one cluster barrier every CTA has its bases and the totals: segment offsets,
//     then the stores -- slot in entry order, the inverse maps and the dedup lists in runs of
//     consecutive addresses (one run per (tile, expert) and per (tile, rank)).
// One grid-wide exchange and one cluster barrier replace the cooperative kernel's two grid
// barriers and its scan phase.  The launch is cooperative (every CTA waits for all others),
// and the host checks that all of its clusters can be resident at once.  The exchange's wait
// gives up after the wait limit; a CTA that gave up still takes every cluster barrier, so no
// barrier of its cluster can hang.
constexpr int kMaxClusterTiles = 16;

// Shared memory of the group kernel after the common layout (words).
struct GroupSmem {
    int32_t *tc;     // [E+R] this tile's counts, then the expert counts of the routing
    int32_t *tb;     // [E+R] this tile's base (earlier tiles), written by the row's owner CTA
    int32_t *tot;    // [E+R] the routing's counts, written by the row's owner CTA
    int32_t *loff;   // [E+1] tile-local first entry of each expert in the staging order
    int32_t *lroff;  // [R+1] tile-local first leader of each rank in the staging order
    int32_t *qloc;   // [kPlanTile * k] each entry's rank among the tile's entries of its expert
    int32_t *lstage; // [kPlanTile * min(k, R)] leaders by (rank, token): rank << 16 | entry
};

__host__ __device__ constexpr size_t plan_group_smem_words(int E, int R, int k)
{
    return plan_smem_words(E, R, k) + 3 * static_cast<size_t>(E + R) + (E + 1) + (R + 1) +
           static_cast<size_t>(kPlanTile) * k + static_cast<size_t>(kPlanTile) * (k < R ? k : R);
}

__device__ __forceinline__ GroupSmem carve_group(const PlanSmem &m, int E, int R, int k)
{
    GroupSmem q;
    const int ER = E + R;
    q.tc = m.end;
    q.tb = q.tc + ER;
    q.tot = q.tb + ER;
    q.loff = q.tot + ER;
    q.lroff = q.loff + E + 1;
    q.qloc = q.lroff + R + 1;
    q.lstage = q.qloc + kPlanTile * k;
    return q;
}

// Split cluster barrier: every thread of every CTA arrives, and later waits for the phase.
__device__ __forceinline__ void cluster_arrive_relaxed()
{
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}

__device__ __forceinline__ void cluster_wait()
{
    asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
}

// Grids of several clusters and up to this many CTAs wait for the exchange while they stage
// their tiles (the kEarlyPoll instantiation); larger ones stage first.
constexpr int kEarlyPollCtas = 256;
// Grids of several clusters with at most kPlanWarps * kLocalRowsPerWarp rows (E + R) and
// 32 * kLocalRounds tiles scan the tile counts in every CTA rather than spreading the rows
// over a cluster and exchanging the results through distributed shared memory.
constexpr int kLocalRowsPerWarp = 4;
constexpr int kLocalRounds = 4;

// kWide: rows of more than 16 ids (k > 16); the other instantiations take k <= 16.
// kEarlyPoll: warp 0 waits for the exchange while warps 1..7 stage the tile (grids of several
// clusters only; a grid of one cluster has no exchange and ignores it).
template <bool kWide, bool kEarlyPoll>
__global__ void __launch_bounds__(kPlanThreads, 4) plan_group_kernel(const PlanK p)
{
    namespace cg = cooperative_groups;
    extern __shared__ __align__(16) int32_t smem[];
    __shared__ uint32_t s_err;
    __shared__ int s_ok;
    __shared__ uint32_t s_gen;  // the exchange generation, read once and shared by the CTA
    cg::cluster_group cluster = cg::this_cluster();
    const PlanSmem m = carve(smem, p.E, p.R, p.k);
    const GroupSmem q = carve_group(m, p.E, p.R, p.k);
    const int ER = p.E + p.R;
    const int k = p.k;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int C = static_cast<int>(cluster.num_blocks());
    const int c = static_cast<int>(cluster.block_rank());
    const int t_first = static_cast<int>(blockIdx.x) - c;  // the cluster's first tile
    const int tile = static_cast<int>(blockIdx.x);
    const int ntok = tile_tokens(p, tile);  // 0 for the CTAs past the last tile

    const bool one_cluster = static_cast<int>(gridDim.x) == C;
    const bool early_poll = kEarlyPoll && !one_cluster;
    // Several clusters but few rows and tiles: every CTA scans the whole table of tile counts.
    const bool local_rows = !one_cluster && ER <= kPlanWarps * kLocalRowsPerWarp &&
                            p.nt <= 32 * kLocalRounds;
    // Arrive at once on the cluster barrier that is waited on before the first access to
    // another CTA's shared memory (every CTA of the cluster has started by then).
    cluster_arrive_relaxed();
    // Shared-memory set-up overlaps the previous kernel on the stream; global memory is
    // touched only after pdl_wait.
    init_rank_of(p, m);
    clear_tile_masks(p, m);
    if (threadIdx.x == 0)
        s_err = 0u;
    pdl_wait();
    load_ids(p, m, tile, ntok);
    if (threadIdx.x == 0) {
        s_gen = __ldcg(&p.sync[1]);
        // Clear the error word before any CTA can or bits into it (all of that happens after
        // the exchange).  A timeout of an earlier call stays until moe_plan_check rearms the
        // plan.
        if (blockIdx.x == 0)
            atomicAnd(p.err, MOE_ERR_TIMEOUT);
    }
    const uint32_t flags = classify_loaded_w<kWide ? 32 : 16>(p, m, ntok);  // syncs first and last
    if (flags)
        atomicOr(&s_err, flags);
    for (int row = threadIdx.x; row < ER; row += blockDim.x) {
        const uint32_t *mk = row < p.E ? &m.emask[4 * row] : &m.rmask[4 * (row - p.E)];
        const int32_t v = __popc(mk[0]) + __popc(mk[1]) + __popc(mk[2]) + __popc(mk[3]);
        q.tc[row] = v;
        if (!one_cluster && tile < p.nt) {
            if (row < p.E)
                p.tile_cnt[static_cast<int64_t>(row) * p.nt + tile] = v;
            else
                p.tile_rcnt[static_cast<int64_t>(row - p.E) * p.nt + tile] = v;
        }
    }
    uint32_t want = s_gen + 1u;  // s_gen was set before classify_loaded's barriers
    if (want == 0u)
        want = 1u;  // arrival words start at 0: the generation never takes that value
    __syncthreads();  // the tile's counts are stored and s_err is final
    if (threadIdx.x == 0 && !one_cluster) {
        if (tile < p.nt)
            p.tile_err[tile] = s_err;
        __threadfence();  // the CTA's stores (ordered before by the barrier) first
        st_release_gpu(&p.group_flag[tile], want);  // every CTA arrives, the last ones too
    }

    // Tile-local offsets and the staging orders (this tile's data only).  With an early poll,
    // warp 0 waits for the arrival words meanwhile and warps 1..7 prepare the tile between
    // themselves (a named barrier joins them).
    const int w0 = early_poll ? 1 : 0;  // first staging warp
    const int n_stage = kPlanWarps - w0;
    if (warp >= w0) {
        if (warp == w0)
            warp_scan_into(q.tc, p.E, q.loff);
        else if (warp == w0 + 1)
            warp_scan_into(q.tc + p.E, p.R, q.lroff);
        if (early_poll)
            asm volatile("bar.sync 1, %0;" ::"r"(n_stage * 32) : "memory");
        else
            __syncthreads();
        const LaneMap lm = lane_map(k);
        const int j = lane & ((1 << lm.wbits) - 1);
        const int sub = lane >> lm.wbits;
        int32_t *estage = m.ids;  // the ids are no longer needed: entries by (expert, token)
        // One (token run, step) pair of the tile.
        auto stage = [&](int vw, int st) {
            const int tw = st * lm.per_step + sub;
            const int tl = vw * kPlanTokensPerWarp + tw;
            if (!(tw < kPlanTokensPerWarp && tl < ntok && j < k))
                return;
            const int i = tl * k + j;
            const int32_t e = m.vid[i];
            if (e < 0)
                return;
            const int32_t r_e = bits_below(&m.emask[4 * e], tl);
            q.qloc[i] = r_e;
            estage[q.loff[e] + r_e] = (e << 16) | i;
            if (m.lead[i] && p.lists) {
                const int32_t r = m.rank_of[e];
                q.lstage[q.lroff[r] + bits_below(&m.rmask[4 * r], tl)] = (r << 16) | i;
            }
        };
        if (!kEarlyPoll) {
            for (int st = 0; st < lm.steps; ++st)  // warp w takes token run w
                stage(warp, st);
        } else {
            // the pairs dealt out round robin to the staging warps
            for (int it = warp - w0; it < kPlanWarps * lm.steps; it += n_stage) {
                const int vw = it / lm.steps;
                stage(vw, it - vw * lm.steps);
            }
        }
    } else {
        // warp 0 of an early poll
        const bool arrived = wait_words_warp(p.group_flag, gridDim.x, want, p.err);
        if (lane == 0)
            s_ok = arrived;
    }
    // The exchange: every CTA's arrival word holds this launch's generation.  A grid of one
    // cluster needs none: its counts are read from the other CTAs' shared memory.
    bool ok = true;
    if (early_poll) {
        __syncthreads();  // warp 0's result
        ok = s_ok != 0;
    } else if (!one_cluster) {
        ok = wait_words(p.group_flag, gridDim.x, want, p.err, &s_ok);
    }
    if (ok && !one_cluster && blockIdx.x == 0 && threadIdx.x == 0)
        p.sync[1] = want;  // every CTA read the old generation before it arrived
    cluster_wait();        // every CTA of the cluster has started (DSMEM is usable)
    if (one_cluster) {
        cluster.sync();  // every tile's counts and flags are in its CTA's shared memory
        // The rows this CTA owns (row % C == c): lane qq of a segment of `width` lanes reads
        // the count of tile qq; a segmented scan gives each tile's base and the total.
        int width = 1;
        while (width < C)
            width <<= 1;
        const int per_warp = 32 / width;
        const int qq = lane & (width - 1);
        const int slot_in_warp = lane / width;
        const int n_own = c < ER ? (ER - c + C - 1) / C : 0;
        for (int i0 = warp * per_warp; i0 < n_own; i0 += kPlanWarps * per_warp) {
            const int i = i0 + slot_in_warp;
            const int row = c + C * i;
            const bool own = i < n_own && qq < C;
            const int32_t v = own ? cluster.map_shared_rank(q.tc, qq)[row] : 0;
            int32_t incl = v;
            for (int o = 1; o < width; o <<= 1) {
                const int32_t y = __shfl_up_sync(kFull, incl, o, width);
                if (qq >= o)
                    incl += y;
            }
            const int32_t total = __shfl_sync(kFull, incl, width - 1, width);
            if (own) {
                cluster.map_shared_rank(q.tb, qq)[row] = incl - v;
                cluster.map_shared_rank(q.tot, qq)[row] = total;
            }
        }
        if (c == 0 && threadIdx.x == 0) {
            uint32_t f = 0u;
            for (int x = 0; x < C; ++x)
                f |= *cluster.map_shared_rank(&s_err, x);
            if (f)
                atomicOr(p.err, f);
        }
    } else if (ok && local_rows) {
        // Few rows and tiles: every CTA reads all of them and takes its own bases and every
        // total itself, with no distributed shared memory and no closing cluster barrier.
        // Warp w takes rows w, w + 8, ...; all of its loads are in flight together.
        int32_t v[kLocalRowsPerWarp][kLocalRounds];
#pragma unroll
        for (int a = 0; a < kLocalRowsPerWarp; ++a) {
            const int row = warp + kPlanWarps * a;
            const int32_t *col = row >= ER    ? nullptr
                                 : row < p.E ? p.tile_cnt + static_cast<int64_t>(row) * p.nt
                                             : p.tile_rcnt + static_cast<int64_t>(row - p.E) * p.nt;
#pragma unroll
            for (int rr = 0; rr < kLocalRounds; ++rr) {
                const int t = rr * 32 + lane;
                v[a][rr] = col != nullptr && t < p.nt ? __ldcg(col + t) : 0;
            }
        }
#pragma unroll
        for (int a = 0; a < kLocalRowsPerWarp; ++a) {
            const int row = warp + kPlanWarps * a;
            int32_t below = 0, total = 0;
#pragma unroll
            for (int rr = 0; rr < kLocalRounds; ++rr) {
                total += v[a][rr];
                below += rr * 32 + lane < tile ? v[a][rr] : 0;
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                total += __shfl_xor_sync(kFull, total, o);
                below += __shfl_xor_sync(kFull, below, o);
            }
            if (row < ER && lane == 0) {
                q.tb[row] = below;
                q.tot[row] = total;
            }
        }
        if (blockIdx.x == 0 && warp == kPlanWarps - 1) {
            uint32_t f = 0u;
            for (int t = lane; t < p.nt; t += 32)
                f |= __ldcg(p.tile_err + t);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
                f |= __shfl_xor_sync(kFull, f, o);
            if (lane == 0 && f)
                atomicOr(p.err, f);
        }
    } else if (ok) {
        // This CTA's rows, one warp per row: a scan over all tiles (coalesced loads of up to
        // kRounds * 32 tiles at a time); each tile of the cluster gets its prefix, and every
        // CTA of the cluster the row's total.
        // A warp takes kRows rows at a time and loads kRounds * 32 tiles of each of them before
        // scanning any, so that its loads are in flight together.
        constexpr int kRows = 3, kRounds = 4;
        const int rpc = (ER + C - 1) / C;
        const int r_lo = c * rpc, r_hi = min(ER, r_lo + rpc);
        for (int rb = r_lo + warp * kRows; rb < r_hi; rb += kPlanWarps * kRows) {
            int32_t carry[kRows];
#pragma unroll
            for (int a = 0; a < kRows; ++a)
                carry[a] = 0;
            for (int t0 = 0; t0 < p.nt; t0 += 32 * kRounds) {
                int32_t v[kRows][kRounds];
#pragma unroll
                for (int a = 0; a < kRows; ++a) {
                    const int row = rb + a;
                    const int32_t *col =
                        row >= r_hi ? nullptr
                        : row < p.E ? p.tile_cnt + static_cast<int64_t>(row) * p.nt
                                    : p.tile_rcnt + static_cast<int64_t>(row - p.E) * p.nt;
#pragma unroll
                    for (int rr = 0; rr < kRounds; ++rr) {
                        const int t = t0 + rr * 32 + lane;
                        v[a][rr] = col != nullptr && t < p.nt ? __ldcg(col + t) : 0;
                    }
                }
#pragma unroll
                for (int a = 0; a < kRows; ++a) {
                    const int row = rb + a;
#pragma unroll
                    for (int rr = 0; rr < kRounds; ++rr) {
                        const int t = t0 + rr * 32 + lane;
                        int32_t incl = v[a][rr];
#pragma unroll
                        for (int o = 1; o < 32; o <<= 1) {
                            const int32_t y = __shfl_up_sync(kFull, incl, o);
                            if (lane >= o)
                                incl += y;
                        }
                        if (row < r_hi && t >= t_first && t < t_first + C && t < p.nt)
                            cluster.map_shared_rank(q.tb, t - t_first)[row] =
                                carry[a] + incl - v[a][rr];
                        carry[a] += __shfl_sync(kFull, incl, 31);
                    }
                }
            }
#pragma unroll
            for (int a = 0; a < kRows; ++a)
                if (rb + a < r_hi && lane < C)
                    cluster.map_shared_rank(q.tot, lane)[rb + a] = carry[a];
        }
        if (blockIdx.x == 0 && warp == kPlanWarps - 1) {
            uint32_t f = 0u;
            for (int t = lane; t < p.nt; t += 32)
                f |= __ldcg(p.tile_err + t);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
                f |= __shfl_xor_sync(kFull, f, o);
            if (lane == 0 && f)
                atomicOr(p.err, f);
        }
    }
    if (local_rows)
        __syncthreads();  // this CTA's bases and totals; no other CTA touches its shared memory
    else
        cluster.sync();  // bases and totals are in place; no DSMEM access after this point
    if (!ok)
        return;
    // Only the output stores remain: let the next kernel on the stream start launching.
    pdl_trigger();

    // Segment sizes are the counts rounded up to the alignment; block 0 publishes the counts.
    for (int e = threadIdx.x; e < p.E; e += blockDim.x) {
        m.ebase[e] = (q.tot[e] + p.align - 1) / p.align * p.align;
        if (blockIdx.x == 0)
            p.cnt[e] = q.tot[e];
    }
    for (int r = threadIdx.x; r < p.R; r += blockDim.x) {
        m.rbase[r] = q.tot[p.E + r];
        if (blockIdx.x == 0)
            p.rcnt[r] = q.tot[p.E + r];
    }
    prepare_offsets(p, m, q.tot, true);  // synchronises first
    if (ntok == 0)
        return;  // block-uniform: a CTA past the last tile has nothing to store
    for (int e = threadIdx.x; e < p.E; e += blockDim.x)
        m.ebase[e] = m.eoff[e] + q.tb[e];
    for (int r = threadIdx.x; r < p.R; r += blockDim.x)
        m.rbase[r] = m.roff[r] + q.tb[p.E + r];
    __syncthreads();

    // The stores: slot in entry order, the inverse maps in (expert, token) order, the dedup
    // lists in (rank, token) order -- consecutive threads write consecutive addresses.
    const int64_t t0 = static_cast<int64_t>(tile) * kPlanTile;
    const int n_ent = ntok * k;
    uint32_t bad = 0u;
    for (int i = threadIdx.x; i < n_ent; i += blockDim.x) {
        const int32_t e = m.vid[i];
        int32_t sv = -1;
        if (e >= 0) {
            sv = m.ebase[e] + q.qloc[i];
            if (static_cast<uint32_t>(sv) >= static_cast<uint32_t>(p.n_rows)) {
                bad |= MOE_ERR_BOUNDS;
                sv = -1;
            }
        }
        p.slot[t0 * k + i] = sv;
    }
    const int32_t n_valid = q.loff[p.E];
    const int32_t *estage = m.ids;
    for (int x = threadIdx.x; x < n_valid; x += blockDim.x) {
        const int32_t v = estage[x];
        const int32_t e = v >> 16, i = v & 0xffff;
        const int32_t sv = m.ebase[e] + (x - q.loff[e]);
        if (static_cast<uint32_t>(sv) < static_cast<uint32_t>(p.n_rows)) {
            p.src_tok[sv] = static_cast<int32_t>(t0 + i / k);
            p.src_j[sv] = i % k;
        }
    }
    const int32_t n_lead = p.lists ? q.lroff[p.R] : 0;
    for (int x = threadIdx.x; x < n_lead; x += blockDim.x) {
        const int32_t v = q.lstage[x];
        const int32_t r = v >> 16, i = v & 0xffff;
        const int32_t pos = m.rbase[r] + (x - q.lroff[r]);
        if (pos >= 0 && pos < p.rtok_cap) {
            p.rtok[pos] = static_cast<int32_t>(t0 + i / k);
            p.fanout[pos] = m.lead[i];
        } else {
            bad |= MOE_ERR_BOUNDS;
        }
    }
    if (bad)
        atomicOr(p.err, bad);
}

// ----------------------------------------------------------- fused (cooperative)

__global__ void __launch_bounds__(kPlanThreads) plan_fused_kernel(const PlanK p)
{
    extern __shared__ __align__(16) int32_t smem[];
    __shared__ uint32_t s_err;
    __shared__ int s_ok;
    const PlanSmem m = carve(smem, p.E, p.R, p.k);
    const uint32_t G = gridDim.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

    init_rank_of(p, m);
    pdl_wait();  // the routing and the plan's arrays are accessed from here on
    uint32_t gen = threadIdx.x == 0 ? ld_acquire_gpu(&p.sync[1]) : 0u;
    for (int tile = blockIdx.x; tile < p.nt; tile += G)
        count_tile(p, m, tile, &s_err);
    if (!grid_barrier(p.sync, p.err, gen, &s_ok))
        return;
    gen += 1u;  // the generation the next barrier starts from

    // Scan phase: one warp per expert row / rank row, in coalesced rounds of 32 tiles;
    // each group of up to 16 rounds is loaded before any of it is scanned.
    constexpr int kRounds = 16;
    for (int row = blockIdx.x * kPlanWarps + warp; row < p.E + p.R;
         row += static_cast<int>(G) * kPlanWarps) {
        int32_t *rp = row < p.E ? p.tile_cnt + static_cast<int64_t>(row) * p.nt
                                : p.tile_rcnt + static_cast<int64_t>(row - p.E) * p.nt;
        int32_t carry = 0;
        for (int g0 = 0; g0 < p.nt; g0 += 32 * kRounds) {
            int32_t v[kRounds];
#pragma unroll
            for (int q = 0; q < kRounds; ++q) {
                const int i = g0 + q * 32 + lane;
                v[q] = i < p.nt ? __ldcg(rp + i) : 0;
            }
#pragma unroll
            for (int q = 0; q < kRounds; ++q) {
                if (g0 + q * 32 < p.nt) {  // warp-uniform
                    const int i = g0 + q * 32 + lane;
                    int32_t incl = v[q];
#pragma unroll
                    for (int o = 1; o < 32; o <<= 1) {
                        const int32_t y = __shfl_up_sync(kFull, incl, o);
                        if (lane >= o)
                            incl += y;
                    }
                    if (i < p.nt)
                        rp[i] = carry + incl - v[q];
                    carry += __shfl_sync(kFull, incl, 31);
                }
            }
        }
        if (lane == 0) {
            if (row < p.E)
                p.cnt[row] = carry;
            else
                p.rcnt[row - p.E] = carry;
        }
    }
    if (blockIdx.x == 0 && warp == 0) {
        uint32_t f = 0;
        for (int i = lane; i < p.nt; i += 32)
            f |= __ldcg(p.tile_err + i);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            f |= __shfl_xor_sync(kFull, f, o);
        if (lane == 0)
            *p.err = f;
    }
    if (!grid_barrier(p.sync, p.err, gen, &s_ok))
        return;
    pdl_trigger();  // only the rank phase remains: let the next kernel start launching

    rank_prepare(p, m);
    // With one tile per CTA the count phase left that tile's classification in smem.
    const bool one_tile = static_cast<int>(G) >= p.nt;
    for (int tile = blockIdx.x; tile < p.nt; tile += G)
        rank_tile(p, m, tile, one_tile);
}

PlanK make_params(const int32_t *topk_idx, int32_t N, int32_t k, int32_t E, int32_t R,
                  int32_t align, int64_t rtok_cap)
{
    PlanK p{};
    p.topk_idx = topk_idx;
    p.N = N;
    p.k = k;
    p.E = E;
    p.R = R;
    p.epr = E / R;
    p.nt = static_cast<int32_t>(ceil_div(N, kPlanTile));
    p.align = align;
    p.n_rows = static_cast<int32_t>(recv_rows(N, k, E, align));
    p.rtok_cap = rtok_cap;
    // Match instructions for the widest rows of ids (k > 16); shuffle compares below that.
    // Measured on B200 at 16384 tokens of 256 experts: k = 32 plans in 42 us with match
    // instructions against 46 with shuffles; at k = 16 the shuffles are faster (26 against
    // 27 us), at k <= 8 clearly so.
    const int mode = tuning().plan_match;
    p.match = mode == 2 ? 1 : mode == 1 ? 0 : (k > 16 ? 1 : 0);
    p.lists = 1;
    return p;
}

bool ensure_attrs(int dev)
{
    static bool done[64] = {false};
    if (dev < 0 || dev >= 64)
        dev = 0;
    if (done[dev])
        return true;
    const int bytes = static_cast<int>(sizeof(int32_t) *
                                       plan_smem_words(kMaxExperts, kMaxExperts, kMaxTopk));
    if (cudaFuncSetAttribute(plan_count_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             bytes) != cudaSuccess ||
        cudaFuncSetAttribute(plan_rank_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             bytes) != cudaSuccess ||
        cudaFuncSetAttribute(plan_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             bytes) != cudaSuccess ||
        cudaFuncSetAttribute(plan_one_tile_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             bytes) != cudaSuccess)
        return false;
    done[dev] = true;
    return true;
}

cudaError_t launch_three(const PlanK &p, int device, cudaStream_t stream)
{
    const size_t smem = sizeof(int32_t) * plan_smem_words(p.E, p.R, p.k);
    cudaError_t e = cudaSuccess;
    if (p.nt > 0)
        e = launch_kernel(plan_count_kernel, dim3(p.nt), dim3(kPlanThreads), smem, stream, false,
                          device, p);
    if (e == cudaSuccess)
        e = launch_kernel(plan_scan_kernel, dim3(p.E + p.R), dim3(kScanThreads), 0, stream,
                          false, device, p);
    if (e == cudaSuccess)
        e = launch_kernel(plan_rank_kernel, dim3(p.nt > 0 ? p.nt : 1), dim3(kPlanThreads), smem,
                          stream, false, device, p);
    return e;
}

}  // namespace

namespace {

// How many clusters of the group kernel, `C` CTAs with `smem` bytes each, can be resident at
// once on `device` (cached: the answer depends only on these).  -1 when the query fails.
int group_clusters_resident(const void *kernel, int C, size_t smem, int device,
                            const cudaLaunchConfig_t *cfg)
{
    struct Fit {
        const void *kernel;
        int C, device;
        size_t smem;
        int clusters;
    };
    static Fit cache[64];
    static int n_cache = 0;
    for (int i = 0; i < n_cache; ++i)
        if (cache[i].kernel == kernel && cache[i].C == C && cache[i].device == device &&
            cache[i].smem == smem)
            return cache[i].clusters;
    int c = 0;
    if (cudaOccupancyMaxActiveClusters(&c, kernel, cfg) != cudaSuccess) {
        (void)cudaGetLastError();
        c = -1;
    }
    if (n_cache < 64)
        cache[n_cache++] = {kernel, C, device, smem, c};
    return c;
}

// The group kernel on `nt` >= 2 tiles, if its clusters can all be resident; false (nothing
// enqueued) otherwise.  Clusters of more than 8 CTAs use the non-portable size that sm_100
// allows.  With several groups the launch is cooperative; if the runtime refuses a
// cooperative cluster launch, the group kernel is not used again on that device.
bool launch_groups(const PlanK &p, int device, cudaStream_t stream, cudaError_t *err)
{
    static int non_portable[64][4] = {};  // per kernel: 1 allowed, -1 refused
    static int coop_clusters[64] = {0};   // -1: a cooperative cluster launch was refused
    const int dv = device >= 0 && device < 64 ? device : 0;
    if (coop_clusters[dv] < 0)
        return false;
    const int wide = p.k > 16 ? 1 : 0;
    const void *const kernels[4] = {reinterpret_cast<const void *>(plan_group_kernel<false, false>),
                                    reinterpret_cast<const void *>(plan_group_kernel<true, false>),
                                    reinterpret_cast<const void *>(plan_group_kernel<false, true>),
                                    reinterpret_cast<const void *>(plan_group_kernel<true, true>)};
    const size_t smem = sizeof(int32_t) * plan_group_smem_words(p.E, p.R, p.k);
    if (smem > static_cast<size_t>(max_smem_optin(device)))
        return false;
    // The kernel's shared-memory limit raised, and its clusters of more than 8 CTAs allowed
    // (false if it cannot run at all; *big false if clusters stay at 8 CTAs at most).
    auto prepare = [&](int which, bool *big) {
        int per_sm = 0;
        if (kernel_fit(kernels[which], device, kPlanThreads, smem, &per_sm) != cudaSuccess ||
            per_sm < 1) {
            (void)cudaGetLastError();
            return false;
        }
        if (non_portable[dv][which] == 0)
            non_portable[dv][which] =
                cudaFuncSetAttribute(kernels[which],
                                     cudaFuncAttributeNonPortableClusterSizeAllowed,
                                     1) == cudaSuccess
                    ? 1
                    : -1;
        if (non_portable[dv][which] < 0)
            (void)cudaGetLastError();
        *big = non_portable[dv][which] > 0;
        return true;
    };
    bool big = false;
    if (!prepare(wide, &big))
        return false;
    const void *kernel = kernels[wide];
    int cmax = tuning().plan_cluster > 0 ? std::min(tuning().plan_cluster, kMaxClusterTiles)
                                         : kMaxClusterTiles;
    if (cmax > 8 && !big)
        cmax = 8;
    // The largest cluster size whose clusters can all be resident at once (16 CTAs of a
    // cluster share one GPC, so a grid of many large clusters may not fit where smaller
    // clusters do).
    int C = 0, G = 0;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    for (int c = std::min(cmax, p.nt); c >= 1 && C == 0; c = c > 8 ? 8 : 0) {
        const int g = static_cast<int>(ceil_div(p.nt, c));
        cfg.gridDim = dim3(static_cast<unsigned>(g * c));
        cfg.blockDim = dim3(kPlanThreads);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = stream;
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = static_cast<unsigned>(c);
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (group_clusters_resident(kernel, c, smem, device, &cfg) >= g) {
            C = c;
            G = g;
        }
    }
    if (C == 0)
        return false;
    if (G > 1 && G * C <= kEarlyPollCtas) {
        // the early-poll instantiation, where it fits the same clusters
        bool big_e = false;
        if (prepare(2 + wide, &big_e) && (C <= 8 || big_e) &&
            group_clusters_resident(kernels[2 + wide], C, smem, device, &cfg) >= G)
            kernel = kernels[2 + wide];
    }
    PlanK arg = p;
    void *args[] = {&arg};
    const cudaError_t e = launch_ex(kernel, args, cfg.gridDim, cfg.blockDim, smem, stream, G > 1,
                                    device, attr, 1);
    if (e != cudaSuccess) {
        (void)cudaGetLastError();
        if (G > 1)
            coop_clusters[dv] = -1;
        return false;
    }
    *err = cudaSuccess;
    return true;
}

}  // namespace

cudaError_t launch_plan(moe_plan_s *pl, const int32_t *topk_idx, cudaStream_t stream)
{
    if (!ensure_attrs(pl->device))
        return cudaGetLastError() != cudaSuccess ? cudaGetLastError() : cudaErrorUnknown;
    PlanK p = make_params(topk_idx, pl->N, pl->k, pl->E, pl->R, pl->align, pl->rtok_cap);
    p.lists = pl->dedup_lists ? 1 : 0;
    p.tile_cnt = pl->tile_cnt;
    p.tile_rcnt = pl->tile_rcnt;
    p.tile_err = pl->tile_err;
    p.cnt = pl->cnt;
    p.expert_off = pl->expert_off;
    p.rcnt = pl->rcnt;
    p.rank_off = pl->rank_off;
    p.rtok_off = pl->rtok_off;
    p.slot = pl->slot;
    p.src_tok = pl->src_tok;
    p.src_j = pl->src_j;
    p.rtok = pl->rtok;
    p.fanout = pl->fanout;
    p.err = pl->err;
    p.sync = pl->sync;
    p.group_flag = pl->group_flag;

    const int engine = tuning().plan_engine;
    if (engine != 2 && p.nt <= 1) {
        // A single tile: one ordinary launch of one CTA.
        const size_t smem = sizeof(int32_t) * plan_smem_words(p.E, p.R, p.k);
        pl->plan_kernels = 1;
        pl->plan_kind = MOE_PLAN_KIND_ONE_TILE;
        return launch_kernel(plan_one_tile_kernel, dim3(1), dim3(kPlanThreads), smem, stream,
                             false, pl->device, p);
    }
    if (engine != 2 && engine != 3) {
        // Groups of up to 16 tiles on thread-block clusters, when they can all be resident.
        cudaError_t e = cudaSuccess;
        if (launch_groups(p, pl->device, stream, &e)) {
            pl->plan_kernels = 1;
            pl->plan_kind = MOE_PLAN_KIND_GROUPS;
            return e;
        }
    }
    if (engine != 2) {
        // One cooperative launch when the grid fits on the device at once.
        static int coop[64] = {0};
        const int dev = pl->device >= 0 && pl->device < 64 ? pl->device : 0;
        if (coop[dev] == 0) {
            int v = 0;
            cudaDeviceGetAttribute(&v, cudaDevAttrCooperativeLaunch, pl->device);
            coop[dev] = v ? 1 : -1;
        }
        const size_t smem = sizeof(int32_t) * plan_smem_words(p.E, p.R, p.k);
        int per_sm = 0;
        if (coop[dev] > 0 &&
            kernel_fit(reinterpret_cast<const void *>(plan_fused_kernel), pl->device,
                       kPlanThreads, smem, &per_sm) == cudaSuccess &&
            per_sm > 0) {
            // One CTA per tile, and at least enough CTAs for one warp per expert / rank row
            // in the scan phase (a few tiles of a wide expert set would otherwise leave each
            // warp dozens of rows, each one dependent round trip to L2).
            const int64_t fit = static_cast<int64_t>(sm_count(pl->device)) * per_sm;
            const int64_t want = std::max<int64_t>(p.nt, ceil_div(p.E + p.R, kPlanWarps));
            const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(want, fit)));
            pl->plan_kernels = 1;
            pl->plan_kind = MOE_PLAN_KIND_COOPERATIVE;
            return launch_kernel(plan_fused_kernel, dim3(grid), dim3(kPlanThreads), smem, stream,
                                 true, pl->device, p);
        }
        (void)cudaGetLastError();
    }
    pl->plan_kernels = 3;
    pl->plan_kind = MOE_PLAN_KIND_THREE;
    return launch_three(p, pl->device, stream);
}

cudaError_t launch_plan_arrays(const PlanArrays &a, cudaStream_t stream)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (!ensure_attrs(dev))
        return cudaGetLastError() != cudaSuccess ? cudaGetLastError() : cudaErrorUnknown;
    PlanK p = make_params(a.topk_idx, a.N, a.k, a.E, a.R, a.align, a.rtok_cap);
    p.tile_cnt = a.tile_cnt;
    p.tile_rcnt = a.tile_rcnt;
    p.tile_err = a.tile_err;
    p.cnt = a.cnt;
    p.expert_off = a.expert_off;
    p.rcnt = a.rcnt;
    p.rank_off = a.rank_off;
    p.rtok_off = a.rtok_off;
    p.slot = a.slot;
    p.src_tok = a.src_tok;
    p.src_j = a.src_j;
    p.rtok = a.rtok;
    p.fanout = a.fanout;
    p.err = a.err;
    p.sync = nullptr;
    return launch_three(p, dev, stream);
}

}  // namespace moe
