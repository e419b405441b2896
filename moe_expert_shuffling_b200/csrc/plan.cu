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
// all phases in one CTA (plan_one_tile_kernel), and one of 2..16 tiles on one thread-block
// cluster with the tile counts shared through distributed shared memory
// (plan_cluster_kernel).
// When the grid cannot be co-resident the phases run as three kernels instead.
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
    int64_t rtok_cap;
    int32_t *tile_cnt, *tile_rcnt;
    uint32_t *tile_err;
    int32_t *cnt, *expert_off, *rcnt, *rank_off, *rtok_off, *slot, *src_tok, *src_j, *rtok;
    uint32_t *fanout, *err;
    uint32_t *sync;  // [2] grid-barrier arrival count (zero at rest) and generation
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
// this lane holds an entry (token in range and column < k).
__device__ __forceinline__ Entry classify(const int32_t *ids, const int32_t *rank_of, int tl,
                                          int j, bool present, int k, int E, int width)
{
    Entry c;
    const int32_t id = present ? ids[tl * k + j] : -1;
    const bool in_range = present && static_cast<uint32_t>(id) < static_cast<uint32_t>(E);
    bool valid = in_range;
    for (int q = 0; q < k; ++q) {
        const int32_t iq = __shfl_sync(kFull, id, q, width);
        if (q < j && iq == id)
            valid = false;
    }
    // -1 marks an entry the router dropped: no row, no contribution, not an error
    c.flags = (present && !in_range && id != -1 ? MOE_ERR_ID_RANGE : 0u) |
              (in_range && !valid ? MOE_ERR_ID_DUP : 0u);
    c.e = valid ? id : -1;
    c.r = valid ? rank_of[id] : -1;
    uint32_t mask = 0;
    bool leader = valid;
    for (int q = 0; q < k; ++q) {
        const int32_t rq = __shfl_sync(kFull, c.r, q, width);
        if (valid && rq == c.r) {
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

// Shared-memory layout of every plan kernel (words).
struct PlanSmem {
    int32_t *eoff;      // [E+1] segment starts of the experts
    int32_t *roff;      // [R+1] starts of the ranks' dedup lists
    int32_t *ebase;     // [E]   tile base per expert; the histogram while counting
    int32_t *rbase;     // [R]   tile base per rank; the rank histogram while counting
    int32_t *rank_of;   // [E]   rank of each expert
    uint32_t *emask;    // [E][4] tokens of the tile on each expert
    uint32_t *rmask;    // [R][4] tokens of the tile on each rank
    int32_t *ids;       // [kPlanTile * k] the tile's routing ids
    int32_t *vid;       // [kPlanTile * k] valid id or -1
    uint32_t *lead;     // [kPlanTile * k] leader masks
};

__host__ __device__ constexpr size_t plan_smem_words(int E, int R, int k)
{
    return static_cast<size_t>(E + 1) + (R + 1) + E + R + E + 4 * E + 4 * R +
           3 * static_cast<size_t>(kPlanTile) * k;
}

__device__ PlanSmem carve(int32_t *w, int E, int R, int k)
{
    PlanSmem m;
    m.eoff = w;
    m.roff = m.eoff + E + 1;
    m.ebase = m.roff + R + 1;
    m.rbase = m.ebase + E;
    m.rank_of = m.rbase + R;
    m.emask = reinterpret_cast<uint32_t *>(m.rank_of + E);
    m.rmask = m.emask + 4 * E;
    m.ids = reinterpret_cast<int32_t *>(m.rmask + 4 * R);
    m.vid = m.ids + kPlanTile * k;
    m.lead = reinterpret_cast<uint32_t *>(m.vid + kPlanTile * k);
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

__device__ void load_ids(const PlanK &p, const PlanSmem &m, int tile, int ntok)
{
    const int32_t *src = p.topk_idx + static_cast<int64_t>(tile) * kPlanTile * p.k;
    for (int i = threadIdx.x; i < ntok * p.k; i += blockDim.x)
        m.ids[i] = __ldg(src + i);
}

// Classify a tile's entries into shared memory: vid/lead per entry, and each token's bit
// in its experts' and ranks' tile masks.  All threads must call; rank_of must be ready.
// Returns this thread's MOE_ERR_* flags.
__device__ uint32_t classify_tile(const PlanK &p, const PlanSmem &m, int tile, int ntok)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int k = p.k;
    for (int i = threadIdx.x; i < 4 * (p.E + p.R); i += blockDim.x)
        m.emask[i] = 0u;  // emask and rmask are contiguous
    load_ids(p, m, tile, ntok);
    __syncthreads();
    const LaneMap lm = lane_map(k);
    const int j = lane & ((1 << lm.wbits) - 1);
    const int sub = lane >> lm.wbits;
    uint32_t flags = 0;
    for (int st = 0; st < lm.steps; ++st) {
        const int tw = st * lm.per_step + sub;           // token within the warp's 16
        const int tl = warp * kPlanTokensPerWarp + tw;
        const bool present = tw < kPlanTokensPerWarp && tl < ntok && j < k;
        const Entry c = classify(m.ids, m.rank_of, tl, j, present, k, p.E, 1 << lm.wbits);
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

// Segment sizes are the counts rounded up to the alignment.  Also marks every receive
// row that no entry maps to (segment padding and rows after the last segment) with -1
// in src_tok/src_j, spread over all CTAs of the grid.
// Segment offsets from m.ebase (segment sizes) and m.rbase (rank counts), which the caller
// has filled; the rest as rank_prepare.
__device__ void prepare_offsets(const PlanK &p, const PlanSmem &m, int32_t *warp_sums);

__device__ void rank_prepare(const PlanK &p, const PlanSmem &m, int32_t *warp_sums)
{
    for (int i = threadIdx.x; i < p.E + p.R; i += blockDim.x) {
        if (i < p.E) {
            const int32_t c = __ldcg(p.cnt + i);
            m.ebase[i] = (c + p.align - 1) / p.align * p.align;
        } else {
            m.rbase[i - p.E] = __ldcg(p.rcnt + (i - p.E));
        }
    }
    prepare_offsets(p, m, warp_sums);
}

__device__ void prepare_offsets(const PlanK &p, const PlanSmem &m, int32_t *warp_sums)
{
    __syncthreads();
    scan_into(m.ebase, p.E, m.eoff, warp_sums);
    scan_into(m.rbase, p.R, m.roff, warp_sums);
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
            const int32_t first = m.eoff[e] + __ldcg(p.cnt + e);
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
            if (msk) {
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
    extern __shared__ int32_t smem[];
    __shared__ uint32_t s_err;
    const PlanSmem m = carve(smem, p.E, p.R, p.k);
    init_rank_of(p, m);
    count_tile(p, m, blockIdx.x, &s_err);
}

__global__ void __launch_bounds__(kScanThreads) plan_scan_kernel(const PlanK p)
{
    __shared__ int32_t warp_sums[kScanThreads / 32];
    __shared__ uint32_t s_err;
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
}

__global__ void __launch_bounds__(kPlanThreads) plan_rank_kernel(const PlanK p)
{
    extern __shared__ int32_t smem[];
    __shared__ int32_t warp_sums[kPlanThreads / 32];
    const PlanSmem m = carve(smem, p.E, p.R, p.k);
    init_rank_of(p, m);
    rank_prepare(p, m, warp_sums);
    rank_tile(p, m, blockIdx.x, false);
}

// ------------------------------------------------------------- one tile (N <= 128)
// Every phase in one CTA: the counts are the popcounts of the single tile's masks, so no
// scratch, no grid barrier and no cooperative launch is needed.
__global__ void __launch_bounds__(kPlanThreads) plan_one_tile_kernel(const PlanK p)
{
    extern __shared__ int32_t smem[];
    __shared__ uint32_t s_err;
    __shared__ int32_t warp_sums[kPlanThreads / 32];
    const PlanSmem m = carve(smem, p.E, p.R, p.k);
    if (threadIdx.x == 0)
        s_err = 0;
    init_rank_of(p, m);
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
    prepare_offsets(p, m, warp_sums);
    // the tile's bases are the segment starts themselves
    for (int e = threadIdx.x; e < p.E; e += blockDim.x)
        m.ebase[e] = m.eoff[e];
    for (int r = threadIdx.x; r < p.R; r += blockDim.x)
        m.rbase[r] = m.roff[r];
    __syncthreads();
    if (ntok > 0)  // block-uniform
        rank_entries(p, m, 0, ntok);
}

// ------------------------------------------- a few tiles on one thread-block cluster
// Routings of 2..kClusterTiles tiles: one CTA per tile in one cluster.  Each CTA counts its
// tile; after the cluster barrier every CTA reads all tiles' counts from the other CTAs'
// shared memory (distributed shared memory) to get its tile base and the totals.  The
// cluster's hardware barrier replaces the grid barriers, and no global scratch is used.
// Every CTA takes the same two barriers whatever its data.  Up to 16 tiles: clusters of
// more than 8 CTAs are opted into (non-portable size, which sm_100 supports); the launch
// falls back to the cooperative kernel when such a cluster cannot be resident.
constexpr int kClusterTiles = 16;

__host__ __device__ constexpr size_t plan_cluster_smem_words(int E, int R, int k)
{
    return plan_smem_words(E, R, k) + 2 * static_cast<size_t>(E + R);
}

__global__ void __launch_bounds__(kPlanThreads) plan_cluster_kernel(const PlanK p)
{
    namespace cg = cooperative_groups;
    extern __shared__ int32_t smem[];
    __shared__ uint32_t s_err;
    __shared__ int32_t warp_sums[kPlanThreads / 32];
    cg::cluster_group cluster = cg::this_cluster();
    const PlanSmem m = carve(smem, p.E, p.R, p.k);
    int32_t *tc = reinterpret_cast<int32_t *>(m.lead + kPlanTile * p.k);  // [E+R] tile counts
    int32_t *tb = tc + (p.E + p.R);                                       // [E+R] tile bases
    const int tile = static_cast<int>(cluster.block_rank());  // the grid is one cluster
    const int C = static_cast<int>(cluster.num_blocks());
    const int ntok = tile_tokens(p, tile);
    if (threadIdx.x == 0)
        s_err = 0;
    init_rank_of(p, m);
    const uint32_t flags = classify_tile(p, m, tile, ntok);  // synchronises first
    if (flags)
        atomicOr(&s_err, flags);
    for (int e = threadIdx.x; e < p.E; e += blockDim.x) {
        const uint32_t *mk = &m.emask[4 * e];
        tc[e] = __popc(mk[0]) + __popc(mk[1]) + __popc(mk[2]) + __popc(mk[3]);
    }
    for (int r = threadIdx.x; r < p.R; r += blockDim.x) {
        const uint32_t *mk = &m.rmask[4 * r];
        tc[p.E + r] = __popc(mk[0]) + __popc(mk[1]) + __popc(mk[2]) + __popc(mk[3]);
    }
    cluster.sync();  // every tile's counts and flags are visible to the cluster

    // this tile's base (earlier tiles) and the total of every expert / rank row
    for (int row = threadIdx.x; row < p.E + p.R; row += blockDim.x) {
        int32_t before = 0, total = 0;
        for (int c = 0; c < C; ++c) {
            const int32_t v = cluster.map_shared_rank(tc, c)[row];
            before += c < tile ? v : 0;
            total += v;
        }
        tb[row] = before;
        // every CTA writes the same totals, so each reads back its own writes below
        if (row < p.E) {
            p.cnt[row] = total;
            m.ebase[row] = (total + p.align - 1) / p.align * p.align;
        } else {
            p.rcnt[row - p.E] = total;
            m.rbase[row - p.E] = total;
        }
    }
    if (tile == 0 && threadIdx.x == 0) {
        uint32_t f = 0;
        for (int c = 0; c < C; ++c)
            f |= *cluster.map_shared_rank(&s_err, c);
        *p.err = f;  // before any MOE_ERR_BOUNDS of the rank step is or-ed in
    }
    cluster.sync();  // no shared memory is read across the cluster after this point

    prepare_offsets(p, m, warp_sums);
    for (int e = threadIdx.x; e < p.E; e += blockDim.x)
        m.ebase[e] = m.eoff[e] + tb[e];
    for (int r = threadIdx.x; r < p.R; r += blockDim.x)
        m.rbase[r] = m.roff[r] + tb[p.E + r];
    __syncthreads();
    rank_entries(p, m, tile, ntok);
}

// ----------------------------------------------------------- fused (cooperative)

__global__ void __launch_bounds__(kPlanThreads) plan_fused_kernel(const PlanK p)
{
    extern __shared__ int32_t smem[];
    __shared__ uint32_t s_err;
    __shared__ int32_t warp_sums[kPlanThreads / 32];
    __shared__ int s_ok;
    const PlanSmem m = carve(smem, p.E, p.R, p.k);
    const uint32_t G = gridDim.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

    uint32_t gen = threadIdx.x == 0 ? ld_acquire_gpu(&p.sync[1]) : 0u;
    init_rank_of(p, m);
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

    rank_prepare(p, m, warp_sums);
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

cudaError_t launch_three(const PlanK &p, cudaStream_t stream)
{
    const size_t smem = sizeof(int32_t) * plan_smem_words(p.E, p.R, p.k);
    if (p.nt > 0)
        plan_count_kernel<<<p.nt, kPlanThreads, smem, stream>>>(p);
    plan_scan_kernel<<<p.E + p.R, kScanThreads, 0, stream>>>(p);
    plan_rank_kernel<<<p.nt > 0 ? p.nt : 1, kPlanThreads, smem, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace

// Whether a cluster of `nt` plan CTAs with `smem` bytes each can be resident (cached: the
// answer depends only on these and the device).
bool cluster_fits(int nt, size_t smem, int device, const cudaLaunchConfig_t *cfg, int *clusters)
{
    struct Fit {
        int nt, device;
        size_t smem;
        int clusters;
    };
    static Fit cache[64];
    static int n_cache = 0;
    for (int i = 0; i < n_cache; ++i)
        if (cache[i].nt == nt && cache[i].device == device && cache[i].smem == smem) {
            *clusters = cache[i].clusters;
            return true;
        }
    int c = 0;
    if (cudaOccupancyMaxActiveClusters(&c, reinterpret_cast<const void *>(plan_cluster_kernel),
                                       cfg) != cudaSuccess)
        return false;
    if (n_cache < 64)
        cache[n_cache++] = {nt, device, smem, c};
    *clusters = c;
    return true;
}

cudaError_t launch_plan(moe_plan_s *pl, const int32_t *topk_idx, cudaStream_t stream)
{
    if (!ensure_attrs(pl->device))
        return cudaGetLastError() != cudaSuccess ? cudaGetLastError() : cudaErrorUnknown;
    PlanK p = make_params(topk_idx, pl->N, pl->k, pl->E, pl->R, pl->align, pl->rtok_cap);
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

    if (tuning().plan_engine != 2 && p.nt <= 1) {
        // A single tile: one ordinary launch of one CTA.
        const size_t smem = sizeof(int32_t) * plan_smem_words(p.E, p.R, p.k);
        pl->plan_kernels = 1;
        plan_one_tile_kernel<<<1, kPlanThreads, smem, stream>>>(p);
        return cudaGetLastError();
    }
    if (tuning().plan_engine != 2 && p.nt <= kClusterTiles) {
        // A few tiles: one cluster of one CTA per tile, when such a cluster can be resident.
        const size_t smem = sizeof(int32_t) * plan_cluster_smem_words(p.E, p.R, p.k);
        int per_sm = 0;
        static int non_portable[64] = {0};
        const int dv = pl->device >= 0 && pl->device < 64 ? pl->device : 0;
        if (non_portable[dv] == 0)
            non_portable[dv] = cudaFuncSetAttribute(plan_cluster_kernel,
                                                    cudaFuncAttributeNonPortableClusterSizeAllowed,
                                                    1) == cudaSuccess ? 1 : -1;
        if ((p.nt <= 8 || non_portable[dv] > 0) &&
            smem <= static_cast<size_t>(max_smem_optin(pl->device)) &&
            kernel_fit(reinterpret_cast<const void *>(plan_cluster_kernel), pl->device,
                       kPlanThreads, smem, &per_sm) == cudaSuccess &&
            per_sm > 0) {
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(static_cast<unsigned>(p.nt));
            cfg.blockDim = dim3(kPlanThreads);
            cfg.dynamicSmemBytes = smem;
            cfg.stream = stream;
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = static_cast<unsigned>(p.nt);
            attr[0].val.clusterDim.y = 1;
            attr[0].val.clusterDim.z = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            int clusters = 0;
            if (cluster_fits(p.nt, smem, pl->device, &cfg, &clusters) && clusters > 0) {
                pl->plan_kernels = 1;
                return cudaLaunchKernelEx(&cfg, plan_cluster_kernel, p);
            }
        }
        (void)cudaGetLastError();
    }
    if (tuning().plan_engine != 2) {
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
            void *args[] = {&p};
            pl->plan_kernels = 1;
            return cudaLaunchCooperativeKernel(reinterpret_cast<const void *>(plan_fused_kernel),
                                               dim3(grid), dim3(kPlanThreads), args, smem, stream);
        }
        (void)cudaGetLastError();
    }
    pl->plan_kernels = 3;
    return launch_three(p, stream);
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
    return launch_three(p, stream);
}

}  // namespace moe
