// Planner: histogram, device-wide prefix scan and stable in-segment rank, plus the
// per-rank dedup lists.  FUSCO (arXiv 2512.22036), abstract: "lightweight planning"
// turns the captured fine-grained layout into placements and removes redundant
// transfers; DySHARP blog, section 5: the destination maps a token's logical index to a
// local address -- slot[t, j] is that map.
//
// Three kernels, all deterministic (no result depends on thread timing):
//   plan_count  one CTA per tile of 128 tokens: per-tile expert counts and per-tile
//               counts of (token, rank) moves -> scratch [E][tiles], [R][tiles]
//   plan_scan   one CTA per expert row and per rank row: exclusive scan over tiles,
//               row totals -> cnt[E], rcnt[R]; CTA 0 also gathers the tile flags
//   plan_rank   one CTA per tile: segment starts, then every entry's stable rank inside
//               its segment as a popcount over a per-expert bitmask of the tile's tokens
//               (bit t set when token t selects the expert), so no step is sequential.
//
// Inside a tile a warp looks at several tokens at once: lane = (token, column) with the
// columns of one token in a segment of W = next power of two >= k lanes, so a token's
// k ids are compared with width-W shuffles.
#include "common.cuh"
#include "internal.cuh"

namespace moe {
namespace {

constexpr int kPlanThreads = kPlanWarps * 32;
constexpr int kScanThreads = 256;
constexpr uint32_t kFull = 0xffffffffu;  // all lanes of a warp

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
    c.flags = (present && !in_range ? MOE_ERR_ID_RANGE : 0u) |
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

__global__ void __launch_bounds__(kPlanThreads)
    plan_count_kernel(const int32_t *__restrict__ topk_idx, int32_t N, int32_t k, int32_t E,
                      int32_t epr, int32_t R, int32_t nt, int32_t *__restrict__ tile_cnt,
                      int32_t *__restrict__ tile_rcnt, uint32_t *__restrict__ tile_err)
{
    extern __shared__ int32_t smem[];
    int32_t *hist = smem;            // [E]
    int32_t *rhist = hist + E;       // [R]
    int32_t *rank_of = rhist + R;    // [E]
    int32_t *ids = rank_of + E;      // [kPlanTile * k]
    __shared__ uint32_t s_err;

    const int tile = blockIdx.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t t0 = static_cast<int64_t>(tile) * kPlanTile;
    const int64_t left = N - t0;
    const int ntok = static_cast<int>(left < kPlanTile ? left : kPlanTile);

    for (int i = threadIdx.x; i < E + R; i += blockDim.x)
        smem[i] = 0;
    for (int e = threadIdx.x; e < E; e += blockDim.x)
        rank_of[e] = e / epr;
    const int32_t *src = topk_idx + t0 * k;
    for (int i = threadIdx.x; i < ntok * k; i += blockDim.x)
        ids[i] = __ldg(src + i);
    if (threadIdx.x == 0)
        s_err = 0;
    __syncthreads();

    const LaneMap lm = lane_map(k);
    const int j = lane & ((1 << lm.wbits) - 1);
    const int sub = lane >> lm.wbits;
    uint32_t flags = 0;
    for (int st = 0; st < lm.steps; ++st) {
        const int tw = st * lm.per_step + sub;           // token within the warp's 16
        const int tl = warp * kPlanTokensPerWarp + tw;
        const bool present = tw < kPlanTokensPerWarp && tl < ntok && j < k;
        const Entry c = classify(ids, rank_of, tl, j, present, k, E, 1 << lm.wbits);
        flags |= c.flags;
        if (c.e >= 0)
            atomicAdd(&hist[c.e], 1);
        if (c.lead)
            atomicAdd(&rhist[c.r], 1);
    }
    if (flags)
        atomicOr(&s_err, flags);
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
    int32_t *ebase = smem;                        // [E+1] segment starts, then tile bases
    int32_t *rbase = ebase + E + 1;               // [R+1]
    int32_t *rank_of = rbase + R + 1;             // [E]
    uint32_t *emask = reinterpret_cast<uint32_t *>(rank_of + E);  // [E][4] tokens per expert
    uint32_t *rmask = emask + 4 * E;              // [R][4] tokens per rank
    int32_t *ids = reinterpret_cast<int32_t *>(rmask + 4 * R);    // [kPlanTile * k]
    int32_t *vid = ids + kPlanTile * k;           // [kPlanTile * k] valid id or -1
    uint32_t *lead = reinterpret_cast<uint32_t *>(vid + kPlanTile * k);  // [kPlanTile * k]
    __shared__ int32_t warp_sums[kPlanThreads / 32];

    const int tile = blockIdx.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t t0 = static_cast<int64_t>(tile) * kPlanTile;
    const int64_t left = N - t0;
    const int ntok = static_cast<int>(left <= 0 ? 0 : (left < kPlanTile ? left : kPlanTile));

    // Segment starts: exclusive scans of the expert and rank totals.
    scan_into(cnt, E, ebase, warp_sums);
    scan_into(rcnt, R, rbase, warp_sums);
    for (int i = threadIdx.x; i < 4 * (E + R); i += blockDim.x)
        emask[i] = 0u;  // emask and rmask are contiguous
    for (int e = threadIdx.x; e < E; e += blockDim.x)
        rank_of[e] = e / epr;
    const int32_t *src = topk_idx + t0 * k;
    for (int i = threadIdx.x; i < ntok * k; i += blockDim.x)
        ids[i] = __ldg(src + i);
    __syncthreads();
    if (tile == 0) {
        for (int i = threadIdx.x; i <= E; i += blockDim.x)
            expert_off[i] = ebase[i];
        for (int i = threadIdx.x; i <= R; i += blockDim.x) {
            rtok_off[i] = rbase[i];
            rank_off[i] = ebase[i * epr];
        }
    }
    if (ntok == 0)
        return;  // block-uniform; no barrier follows for this block
    __syncthreads();
    // This tile's first receive row per expert and first dedup entry per rank.
    for (int e = threadIdx.x; e < E; e += blockDim.x)
        ebase[e] += tile_cnt[static_cast<int64_t>(e) * nt + tile];
    for (int r = threadIdx.x; r < R; r += blockDim.x)
        rbase[r] += tile_rcnt[static_cast<int64_t>(r) * nt + tile];

    // Pass A: classify, and mark each token in its expert's and rank's tile mask.
    const LaneMap lm = lane_map(k);
    const int j = lane & ((1 << lm.wbits) - 1);
    const int sub = lane >> lm.wbits;
    for (int st = 0; st < lm.steps; ++st) {
        const int tw = st * lm.per_step + sub;
        const int tl = warp * kPlanTokensPerWarp + tw;
        const bool present = tw < kPlanTokensPerWarp && tl < ntok && j < k;
        const Entry c = classify(ids, rank_of, tl, j, present, k, E, 1 << lm.wbits);
        if (present) {
            vid[tl * k + j] = c.e;
            lead[tl * k + j] = c.lead;
            const uint32_t bit = 1u << (tl & 31);
            if (c.e >= 0)
                atomicOr(&emask[4 * c.e + (tl >> 5)], bit);
            if (c.lead)
                atomicOr(&rmask[4 * c.r + (tl >> 5)], bit);
        }
    }
    __syncthreads();

    // Pass B: stable rank = tile base + earlier tokens of the tile on the same expert.
    uint32_t flags = 0;
    for (int st = 0; st < lm.steps; ++st) {
        const int tw = st * lm.per_step + sub;
        const int tl = warp * kPlanTokensPerWarp + tw;
        if (!(tw < kPlanTokensPerWarp && tl < ntok && j < k))
            continue;
        const int64_t t = t0 + tl;
        const int i = tl * k + j;
        const int32_t e = vid[i];
        int32_t s = -1;
        if (e >= 0) {
            s = ebase[e] + bits_below(&emask[4 * e], tl);
            if (static_cast<uint32_t>(s) < static_cast<uint32_t>(n_rows)) {
                src_tok[s] = static_cast<int32_t>(t);
                src_j[s] = j;
            } else {
                flags |= MOE_ERR_BOUNDS;
                s = -1;
            }
            const uint32_t m = lead[i];
            if (m) {
                const int32_t r = rank_of[e];
                const int32_t pos = rbase[r] + bits_below(&rmask[4 * r], tl);
                if (pos >= 0 && pos < rtok_cap) {
                    rtok[pos] = static_cast<int32_t>(t);
                    fanout[pos] = m;
                } else {
                    flags |= MOE_ERR_BOUNDS;
                }
            }
        }
        slot[t * k + j] = s;
    }
    if (flags)
        atomicOr(err, flags);
}

size_t count_smem(int E, int R, int k) { return sizeof(int32_t) * (2 * E + R + kPlanTile * k); }
size_t rank_smem(int E, int R, int k)
{
    return sizeof(int32_t) * ((E + 1) + (R + 1) + E + 4 * (E + R) + 3 * kPlanTile * k);
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

cudaError_t launch_plan_arrays(const PlanArrays &a, cudaStream_t stream)
{
    static bool attrs_set[64] = {false};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (dev < 0 || dev >= 64)
        dev = 0;
    if (!attrs_set[dev]) {
        const int max_rank = static_cast<int>(rank_smem(kMaxExperts, kMaxExperts, kMaxTopk));
        const int max_count = static_cast<int>(count_smem(kMaxExperts, kMaxExperts, kMaxTopk));
        e = cudaFuncSetAttribute(plan_rank_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 max_rank);
        if (e != cudaSuccess)
            return e;
        e = cudaFuncSetAttribute(plan_count_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 max_count);
        if (e != cudaSuccess)
            return e;
        attrs_set[dev] = true;
    }
    const int32_t N = a.N, k = a.k, E = a.E, R = a.R, epr = E / R;
    const int32_t nt = static_cast<int32_t>(ceil_div(N, kPlanTile));
    if (nt > 0) {
        plan_count_kernel<<<nt, kPlanThreads, count_smem(E, R, k), stream>>>(
            a.topk_idx, N, k, E, epr, R, nt, a.tile_cnt, a.tile_rcnt, a.tile_err);
    }
    plan_scan_kernel<<<E + R, kScanThreads, 0, stream>>>(a.tile_cnt, a.tile_rcnt, E, R, nt, a.cnt,
                                                          a.rcnt, a.tile_err, a.err);
    plan_rank_kernel<<<nt > 0 ? nt : 1, kPlanThreads, rank_smem(E, R, k), stream>>>(
        a.topk_idx, N, k, E, epr, R, nt, a.tile_cnt, a.tile_rcnt, a.cnt, a.rcnt, a.expert_off,
        a.rank_off, a.rtok_off, a.slot, a.src_tok, a.src_j, a.rtok, a.fanout, N * k, a.rtok_cap,
        a.err);
    return cudaGetLastError();
}

}  // namespace moe
