// Combine: out[t] = bf16_rne( fp32 fma chain over j = 0..k-1 of w[t, j] * y[slot[t, j]] ),
// starting from +0 -- the expert results of a token brought back and summed (DySHARP blog,
// sections 1-2).  The chain runs in top-k column order, so every launch configuration
// gives the same bits.
//
// Bulk-copy engine (combine_cta.cuh): CTAs of one producer warp and CW consumer
// warps (8, 4, 2 or 1 as k grows), each CTA taking a short run of tokens on a grid that
// covers them all.  Work unit = (token, CW * 512-byte column chunk of every row).  The
// producer issues one bulk async copy per routed row chunk (lane j copies row slot[t, j])
// into a ring of stages in shared memory, each completing on a "full" mbarrier; consumers
// take a stage, each thread reduces 8 columns over the k rows from shared memory and
// writes 16 bytes of out, then release the stage on its "empty" mbarrier.  Bytes in flight
// are bounded by shared memory rather than by registers.
#include <algorithm>

#include "combine_cta.cuh"
#include "common.cuh"
#include "internal.cuh"

namespace moe {
namespace {

// Measured on B200 (dsv3 and long shapes): a ring of 32-36 KB per CTA, 3 CTAs per SM and
// short runs of tokens per CTA (the block scheduler evens out the tail) are fastest;
// deeper rings, more CTAs per SM and persistent CTAs are slower.  A run moves about 256 KB
// of rows: graph-replayed steps of the DeepSeek-V3 shape (129 KB per token) took 651 us with
// runs of 2 tokens against 659 us with 4; top-16 (244 KB per token) 1211 against 1226 us and
// top-32 (473 KB) 2381 against 2422 us with runs of 1 token against 4; long context (57 KB)
// is the same from 2 to 4 tokens.  The wide shape for k <= 4 (Mixtral, 24 KB per token)
// starts from runs of 8 tokens.
constexpr int kDefaultSmemBudget = 36 * 1024 + 128;
constexpr int kDefaultCtasPerSm = 3;
constexpr int kDefaultTokensPerCta = 4;
constexpr int64_t kRunTargetBytes = 256 * 1024;
// Below this many waves of resident CTAs the runs change length to fill whole waves, up to
// kMaxRunBytes of rows read and written per run.  Measured on B200 at the Mixtral shape
// (k = 2, 24 KB per token; graph-replayed steps): 8192 tokens 75.0 -> 71.8 us, 4096 tokens
// 40.8 -> 39.0 us, 2048 tokens 27.7 -> 22.3 us.  At the DeepSeek-V3 shape a run of 4 tokens
// already moves 516 KB, and longer runs were slower (4096 tokens: 186.6 against 189.0 us).
constexpr int64_t kWholeWavesBelow = 3;
constexpr int64_t kMaxRunBytes = 512 * 1024;

template <int KMAX, int CW, bool RANKED>
__global__ void __launch_bounds__(Shape<CW>::kThreads, CW >= 8 ? 2 : 1)
    combine_bulk_kernel(const CombineBulkParams p)
{
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    CombineRing r;
    r.carve<RANKED>(p, smem, warp);

    // this CTA's first token, and the range of chunks it takes of each (csplit CTAs share a
    // run of tokens when there are few tokens)
    const uint32_t b = blockIdx.x / p.csplit * p.per_cta;
    const uint32_t cpg = (p.nchunks + p.csplit - 1) / p.csplit;
    const uint32_t c_lo = blockIdx.x % p.csplit * cpg;
    const uint32_t c_hi = min(p.nchunks, c_lo + cpg);
    const int n_tok = b < static_cast<uint32_t>(p.N)
                          ? static_cast<int>(min(p.per_cta, static_cast<uint32_t>(p.N) - b))
                          : 0;
    if (threadIdx.x == 0)
        r.init<CW>();
    pdl_trigger();
    pdl_wait();  // the plan and the expert outputs are read from here on
    // the first token's slots (and, for the consumers, weights) are fetched before the
    // barrier so that their latency overlaps the set-up
    int32_t s_first = -1;
    float w_first = 0.f;
    if (n_tok > 0 && lane < p.k) {
        s_first = __ldg(p.slot + static_cast<int64_t>(b) * p.k + lane);
        if (warp > 0)
            w_first = __ldg(p.w + static_cast<int64_t>(b) * p.k + lane);
    }
    if (RANKED)
        for (int q = threadIdx.x; q <= p.R; q += blockDim.x)
            r.roff_s[q] = __ldg(p.rank_off + q);
    __syncthreads();

    int i = 0;
    if (warp == 0)
        (void)combine_produce<KMAX, CW, RANKED>(p, r, b, n_tok, s_first, i, nullptr, 0u, c_lo,
                                                c_hi);
    else
        (void)combine_consume<KMAX, CW, RANKED>(p, r, b, n_tok, s_first, w_first, i, c_lo, c_hi);
}

}  // namespace

template <int KMAX, int CW, bool RANKED>
cudaError_t launch_bulk_shape(const CombineArgs &a, int device, cudaStream_t stream)
{
    constexpr uint32_t chunk = Shape<CW>::kChunk;
    constexpr int threads = Shape<CW>::kThreads;
    const Tuning &tu = tuning();
    CombineBulkParams p;
    p.y = reinterpret_cast<const uint8_t *>(a.y);
    p.slot = a.slot;
    p.w = a.w;
    p.out = reinterpret_cast<uint8_t *>(a.out);
    p.err = a.err;
    p.N = a.N;
    p.k = a.k;
    p.n_rows = a.n_rows;
    p.row_bytes = static_cast<uint32_t>(a.H) * 2u;
    p.nchunks = static_cast<uint32_t>(ceil_div(p.row_bytes, chunk));
    p.stage_bytes = static_cast<uint32_t>(a.k) * chunk;

    const int max_optin = max_smem_optin(device);
    cudaError_t e = cudaSuccess;
    // Several CTAs per SM (more consumer warps) beat one CTA with a deeper ring.
    const int budget = tu.combine_smem_kb > 0 ? std::min(tu.combine_smem_kb * 1024, max_optin)
                                              : std::min(kDefaultSmemBudget, max_optin);
    int S = tu.combine_stages > 0 ? tu.combine_stages : kMaxBulkStages;
    S = std::min(S, kMaxBulkStages);
    p.rank_off = a.rank_off;
    p.R = a.R;
    // rank-grouped order: the rank offsets plus 64 words per consumer warp
    const size_t tables = RANKED ? sizeof(int32_t) * (static_cast<size_t>(a.R) + 1 + 64 * CW) : 0;
    auto smem_for = [&](int st) {
        return static_cast<size_t>(round_up(2 * st * 8, 128)) +
               static_cast<size_t>(st) * p.stage_bytes + tables;
    };
    // the budget is for the ring; the ranked order's tables come on top of it
    while (S > 2 && smem_for(S) - tables > static_cast<size_t>(budget))
        --S;
    if (smem_for(S) > static_cast<size_t>(max_optin))
        return cudaErrorInvalidValue;
    p.stages = static_cast<uint32_t>(S);
    p.bar_bytes = static_cast<uint32_t>(round_up(2 * S * 8, 128));
    p.ring_bytes = static_cast<uint32_t>(S) * p.stage_bytes;
    const size_t smem = smem_for(S);
    auto kern = combine_bulk_kernel<KMAX, CW, RANKED>;
    int per_sm = 0;
    e = kernel_fit(reinterpret_cast<const void *>(kern), device, threads, smem, &per_sm);
    if (e != cudaSuccess)
        return e;
    if (per_sm < 1)
        return cudaErrorInvalidConfiguration;
    // CTAs the device holds at once (what the block scheduler runs as one wave)
    const int64_t wave = static_cast<int64_t>(sm_count(device)) * per_sm;
    // the default keeps about 12 consumer warps per SM whatever the chunk width
    per_sm = std::min(per_sm, tu.combine_ctas_per_sm > 0 ? tu.combine_ctas_per_sm
                                                          : std::max(1, kDefaultCtasPerSm * 4 / CW));
    // Contiguous runs of tokens per CTA; the grid covers all tokens so that CTAs that
    // finish early are replaced by the block scheduler.
    const int64_t resident = static_cast<int64_t>(sm_count(device)) * per_sm;
    // A run moves about kRunTargetBytes (at most kDefaultTokensPerCta tokens) in the shapes
    // for k > 4, and 2 * kDefaultTokensPerCta tokens in the wide shape for k <= 4.
    const int64_t token_bytes = 2LL * a.H * (a.k + 1);
    int64_t per_cta = 2 * kDefaultTokensPerCta;
    if (tu.combine_tokens_per_cta > 0)
        per_cta = tu.combine_tokens_per_cta;
    else if (CW < 8)
        per_cta = std::min<int64_t>(kDefaultTokensPerCta,
                                    std::max<int64_t>(1, (kRunTargetBytes + token_bytes / 2) /
                                                             token_bytes));
    if (ceil_div(a.N, per_cta) < resident) {
        per_cta = std::max<int64_t>(1, ceil_div(a.N, resident));
    } else if (tu.combine_tokens_per_cta == 0 && ceil_div(a.N, per_cta) < kWholeWavesBelow * wave) {
        // Fewer than three waves: a last wave that is partly empty costs a large share of the
        // kernel, so the runs change length until the grid fills whole waves (the count of
        // waves rounded down; less than one wave is shortened to fill one), as long as a run
        // moves at most kMaxRunBytes.
        const int64_t waves = std::max<int64_t>(1, ceil_div(a.N, per_cta) / wave);
        const int64_t t = ceil_div(a.N, waves * wave);
        if (t * token_bytes <= kMaxRunBytes)
            per_cta = t;
    }
    p.per_cta = static_cast<uint32_t>(per_cta);
    int64_t grid = std::max<int64_t>(1, ceil_div(a.N, per_cta));
    // Few tokens (a decode-sized batch): several CTAs share each run of tokens, each taking a
    // range of the column chunks, so that the SMs do not idle while a handful of CTAs walk
    // whole rows.
    // The split is resident / grid rounded to nearest: rounding up could spill a grid that
    // nearly fills the device into a second, mostly idle wave (measured at 1024 tokens of the
    // dsv3 shape: 26.6 us split in two against 23.3 us unsplit).
    int64_t csplit = 1;
    if (tu.combine_split != 1 && grid < resident && p.nchunks > 1) {
        csplit = std::min<int64_t>(p.nchunks, std::max<int64_t>(1, (2 * resident + grid) / (2 * grid)));
        if (tu.combine_split > 1)
            csplit = std::min<int64_t>(csplit, tu.combine_split);
    }
    p.csplit = static_cast<uint32_t>(csplit);
    grid *= csplit;
    return launch_kernel(kern, dim3(static_cast<unsigned>(grid)), dim3(threads), smem, stream,
                         false, device, p);
}

template <bool RANKED>
cudaError_t launch_combine_bulk(const CombineArgs &a, int device, cudaStream_t stream)
{
    // Chunks widen for k <= 4 (8 consumer warps, 4 KB per row) so that a stage is not a
    // couple of 2 KB rows with a barrier round each.  Measured on B200 at the Mixtral
    // shape (k = 2): 35.6 us against 49.7 us with 4 consumer warps; 16 consumer warps
    // (8 KB per row) were slower than 8.
    const int max_cw = tuning().combine_max_cw > 0 ? tuning().combine_max_cw : 8;
    if (a.k <= 4 && max_cw >= 8)
        return launch_bulk_shape<4, 8, RANKED>(a, device, stream);
    if (a.k <= 8)
        return launch_bulk_shape<8, 4, RANKED>(a, device, stream);
    if (a.k <= 16)
        return launch_bulk_shape<16, 2, RANKED>(a, device, stream);
    return launch_bulk_shape<32, 1, RANKED>(a, device, stream);
}

cudaError_t launch_combine(const CombineArgs &a, int device, cudaStream_t stream)
{
    if (a.N == 0)
        return cudaSuccess;
    if (a.ranked)
        return launch_combine_bulk<true>(a, device, stream);
    return launch_combine_bulk<false>(a, device, stream);
}

}  // namespace moe
