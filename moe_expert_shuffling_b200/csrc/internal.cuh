// Host-side internals shared by the C ABI (api.cu) and the kernel launchers.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "moe_shuffle.h"

// Plan object behind moe_plan_t.  All arrays live in one device allocation.
struct moe_plan_s {
    int32_t cap = 0;        // largest N accepted
    int32_t N = 0, k = 0, E = 0, R = 0, epr = 0;
    int32_t align = 1;      // expert segments start on multiples of this many rows
    bool dedup_lists = true;  // moe_plan writes rtok / fanout
    int32_t nt_cap = 0;     // tiles for `cap` tokens
    int64_t rtok_cap = 0;   // entries of rtok/fanout: cap * min(k, R)
    int64_t rows_cap = 0;   // receive rows for `cap` tokens: cap * k + E * (align - 1)
    int device = 0;
    void *mem = nullptr;
    size_t mem_bytes = 0;
    // outputs
    int32_t *cnt = nullptr, *expert_off = nullptr, *rcnt = nullptr, *rank_off = nullptr,
            *rtok_off = nullptr, *slot = nullptr, *src_tok = nullptr, *src_j = nullptr,
            *rtok = nullptr;
    uint32_t *fanout = nullptr, *err = nullptr;
    uint32_t *sync = nullptr;  // [2] grid-barrier words of the fused plan kernel (zero at rest)
    // scratch: per-tile counts [E][nt] and [R][nt] (then their column prefixes), tile flags
    // (the group kernel keeps its groups' totals and flags in the first rows of these)
    int32_t *tile_cnt = nullptr, *tile_rcnt = nullptr;
    uint32_t *tile_err = nullptr;
    uint32_t *group_flag = nullptr;  // [nt + 16] arrival words of the group plan kernel's CTAs
    const float *topk_w = nullptr;
    int32_t plan_kernels = 0;  // kernels the last launch_plan enqueued
    int32_t plan_kind = 0;     // MOE_PLAN_KIND_* of the last launch_plan
    // moe_dispatch_combine: work words [next dispatch item, next combine item, CTAs done,
    // epoch of the last launch] (the launch's last CTA resets the counters and advances the
    // epoch) and per-token ready flags [cap] holding the epoch of the launch that last
    // dispatched the token
    uint32_t *work = nullptr, *ready = nullptr;
};

namespace moe {

// Receive rows of a plan: N * k entries plus up to align - 1 padding rows per expert.
inline int64_t recv_rows(int64_t N, int32_t k, int32_t E, int32_t align)
{
    return N * k + static_cast<int64_t>(E) * (align - 1);
}

// Tokens per plan tile (one CTA of the count and rank kernels).
constexpr int kPlanWarps = 8;
constexpr int kPlanTokensPerWarp = 16;
constexpr int kPlanTile = kPlanWarps * kPlanTokensPerWarp;
constexpr int kMaxExperts = 1024;
constexpr int kMaxTopk = 32;

// Tunable launch parameters (0 = built-in default).  Set through moe_tune.
struct Tuning {
    int dispatch_stages = 0;
    int dispatch_lag = 0;
    int dispatch_ctas_per_sm = 0;
    int dispatch_warps_per_cta = 0;
    int combine_ctas_per_sm = 0;
    int combine_stages = 0;
    int combine_smem_kb = 0;
    int dispatch_units_per_warp = 0;
    int combine_tokens_per_cta = 0;
    int plan_engine = 0;       // 0/1: automatic, 2: three kernels, 3: no cluster kernel
    int fused_ctas_per_sm = 0;
    int fused_dispatch_share = 0;  // percent of CTAs that start on dispatch work
    int fused_dispatch_run = 0;    // tokens per dispatch work item
    int fused_combine_run = 0;     // tokens per combine work item
    int fused_smem_kb = 0;
    int fused_min_kb = 0;          // least traffic for the one-launch kernel
    int combine_max_cw = 0;        // cap on consumer warps per combine CTA (4, 8 or 16)
    int plan_cluster = 0;          // most tiles per cluster of the group plan kernel (1..16)
    int pdl = 0;                   // 0/1: programmatic dependent launch, 2: ordinary launches
    int plan_match = 0;            // 0: by k, 1: shuffle compares, 2: warp match instructions
    int dispatch_split_units = 0;  // 0: automatic, 1: never cut rows finer, n: below n units
    int combine_split = 0;         // 0: automatic, 1: never split a token's chunks, n: at most n
};
Tuning &tuning();

int sm_count(int device);

// Launch `kernel` with cudaLaunchKernelEx, as a programmatic dependent launch (the kernel
// may begin while the previous kernel on the stream finishes; the kernels wait with
// pdl_wait before touching global memory) unless MOE_TUNE_PDL turns it off, and
// cooperatively when asked.  If the runtime refuses the programmatic attribute for a kind
// of launch on a device, that kind is launched without it from then on.
cudaError_t launch_ex(const void *kernel, void **args, dim3 grid, dim3 block, size_t smem,
                      cudaStream_t stream, bool cooperative, int device,
                      const cudaLaunchAttribute *extra = nullptr, int n_extra = 0);

template <typename... KArgs>
cudaError_t launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                          cudaStream_t stream, bool cooperative, int device, KArgs... args)
{
    void *ptrs[] = {static_cast<void *>(&args)..., nullptr};
    return launch_ex(reinterpret_cast<const void *>(kernel), ptrs, grid, block, smem, stream,
                     cooperative, device);
}

// Largest dynamic shared memory a CTA may opt into on `device` (cached).
int max_smem_optin(int device);

// Resident CTAs per SM of `kernel` with `threads` threads and `smem` bytes of dynamic shared
// memory on `device`, raising the kernel's dynamic-shared-memory limit when needed.  Cached
// per (kernel, device, threads, smem) so that repeated launches make no runtime queries.
cudaError_t kernel_fit(const void *kernel, int device, int threads, size_t smem, int *per_sm);

cudaError_t launch_plan(moe_plan_s *p, const int32_t *topk_idx, cudaStream_t stream);

// The planner's kernels on explicit arrays (for callers that own every buffer).  The
// scratch arrays hold E*tiles, R*tiles and tiles words, tiles = ceil(N / kPlanTile).
struct PlanArrays {
    const int32_t *topk_idx;
    int32_t N, k, E, R;
    int32_t align = 1;
    int64_t rtok_cap;
    int32_t *cnt, *expert_off, *rcnt, *rank_off, *rtok_off, *slot, *src_tok, *src_j, *rtok;
    uint32_t *fanout, *err;
    int32_t *tile_cnt, *tile_rcnt;
    uint32_t *tile_err;
};
cudaError_t launch_plan_arrays(const PlanArrays &a, cudaStream_t stream);

// Record a failure for moe_last_error() and return `st`.
moe_status record_error(moe_status st, const char *fmt, ...);

struct DispatchArgs {
    const uint8_t *x;      // [N, row_bytes]
    const uint8_t *xs;     // [N, srow_bytes] or null
    uint8_t *recv;         // [n_rows, row_bytes]
    uint8_t *rs;           // [n_rows, srow_bytes] or null
    const int32_t *slot;   // [N*k]
    uint32_t *err;
    int32_t N, k, n_rows;
    uint32_t row_bytes, srow_bytes;
};
cudaError_t launch_dispatch(const DispatchArgs &a, int device, cudaStream_t stream);

struct CombineArgs {
    const uint16_t *y;     // bf16 [n_rows, H]
    const int32_t *slot;   // [N*k]
    const float *w;        // [N*k]
    uint16_t *out;         // bf16 [N, H]
    uint32_t *err;
    int32_t N, k, n_rows, H;
    const int32_t *rank_off = nullptr;  // [R+1], for the rank-grouped order
    int32_t R = 0;
    bool ranked = false;   // rank-grouped summation order instead of one chain
};
cudaError_t launch_combine(const CombineArgs &a, int device, cudaStream_t stream);

// One persistent launch doing a dispatch and a combine at once (moe_dispatch_combine).
struct FusedArgs {
    DispatchArgs d;
    CombineArgs c;
    uint32_t *work;          // [4] the dispatch plan's work counters and epoch
    uint32_t *ready;         // [ready_len] the dispatch plan's per-token flags
    uint32_t ready_len;
    bool use_flags;          // c reads the rows d writes (y == recv, one plan)
};
cudaError_t launch_fused(const FusedArgs &a, int device, cudaStream_t stream);

// moe_wait_selftest: one bounded device wait on something that never completes; *flags gets
// the error word (synchronous).
cudaError_t run_wait_selftest(int which, cudaStream_t stream, uint32_t *flags);

}  // namespace moe
