/*
 * moe_shuffle.h -- C ABI of the B200 MoE token-shuffle library (libmoeshuffle.so).
 *
 * The library moves token rows between a token-major layout and an expert-major,
 * rank-segmented layout on one GPU, with the layout change done inside the data
 * movement (FUSCO, arXiv 2512.22036, abstract: the expert-major layout of MoE conflicts
 * with the device-major layout communication expects, so the shuffle is fused into the
 * move).  Expert-parallel ranks are logical: rank r owns the contiguous receive rows of
 * experts r*E/R .. (r+1)*E/R - 1 in one buffer in this GPU's memory.
 *
 * Conventions for every call:
 *   - Pointers named "device" are CUDA device pointers on the current device.  Payload
 *     arrays (x, recv, y, out) must be 16-byte aligned, routing arrays 4-byte aligned.
 *     Arrays are dense and row-major.  A plan is used on the device it was created on.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).
 *     Calls only enqueue work on it; none of them synchronises the host or copies
 *     device data to the host, except moe_plan_check and moe_wait_selftest.
 *   - Arguments are checked on the host before anything is enqueued; a bad argument
 *     returns MOE_EINVAL and enqueues nothing.  A CUDA failure returns MOE_ECUDA.
 *     moe_last_error() then describes the failure (per host thread).
 *   - Routing ids are checked on the device: an id outside [0,E) or an id repeated
 *     within one token sets a bit in the plan's error word (read with moe_plan_check);
 *     the affected entries get slot -1 and are skipped by dispatch and combine, so bad
 *     routing never makes a kernel touch memory outside the caller's buffers.
 *
 * Limits: 1 <= k <= 32, k <= E <= 1024, E % R == 0, 0 <= N, N*k < 2^31.
 */
#ifndef MOE_SHUFFLE_H
#define MOE_SHUFFLE_H

#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MOE_OK = 0,
    MOE_EINVAL = 1,  /* bad argument; nothing was enqueued */
    MOE_ECUDA = 2,   /* a CUDA runtime call or kernel launch failed */
    MOE_ENOMEM = 3   /* device allocation failed */
} moe_status;

typedef enum {
    MOE_BF16 = 0,    /* 2-byte rows; H % 8 == 0 */
    MOE_FP8E4M3 = 1  /* 1-byte rows plus one fp32 scale per 128 columns; H % 128 == 0 */
} moe_dtype;

/* Bits of the plan's device error word. */
#define MOE_ERR_ID_RANGE 1u   /* a routing id outside [0, E) */
#define MOE_ERR_ID_DUP 2u     /* a token listed the same expert twice */
#define MOE_ERR_BOUNDS 4u     /* an internal index fell outside its array (entry skipped) */
#define MOE_ERR_TIMEOUT 8u    /* a device wait gave up after its limit (about 1 s) */

/* Opaque plan: device arrays owned by the library, reusable across calls. */
typedef struct moe_plan_s *moe_plan_t;

/* Device pointers into a plan (valid until moe_plan_destroy; contents valid once the
 * stream of the last moe_plan call has reached that point). */
typedef struct {
    int32_t N, k, E, R;            /* shape of the last moe_plan call */
    int32_t experts_per_rank;      /* E / R */
    int32_t capacity_tokens;       /* largest N this plan accepts */
    int32_t *cnt;                  /* [E]    entries routed to each expert */
    int32_t *expert_off;           /* [E+1]  first receive row of each expert segment */
    int32_t *rcnt;                 /* [R]    tokens that touch rank r (dedup moves) */
    int32_t *rank_off;             /* [R+1]  first receive row of each rank */
    int32_t *rtok_off;             /* [R+1]  start of each rank's dedup list */
    int32_t *slot;                 /* [N*k]  receive row of entry (t, j); -1 if dropped/invalid */
    int32_t *src_tok;              /* [recv_rows] token of each receive row, -1 if none */
    int32_t *src_j;                /* [recv_rows] top-k column of each receive row, -1 if none */
    int32_t *rtok;                 /* [sum rcnt] tokens of rank r, ascending */
    uint32_t *fanout;              /* [sum rcnt] bit j: column j of that token is on rank r */
    uint32_t *err;                 /* [1]    MOE_ERR_* bits of the last moe_plan call */
    const float *topk_w;           /* the weights given to the last moe_plan call */
    int32_t plan_kernels;          /* kernels the last moe_plan call enqueued (1 or 3) */
    int32_t align;                 /* expert segments start on multiples of this many rows */
    int32_t recv_rows;             /* rows a receive buffer needs: N*k + E*(align-1) */
    int32_t plan_kind;             /* MOE_PLAN_KIND_* of the last moe_plan call */
    int32_t dedup_lists;           /* 1 if moe_plan writes rtok / fanout (the default) */
} moe_plan_view;

/* Which planner kernel the last moe_plan call ran (moe_plan_view.plan_kind). */
#define MOE_PLAN_KIND_ONE_TILE 0    /* N <= 128: one block */
#define MOE_PLAN_KIND_GROUPS 1      /* thread-block clusters of up to 16 tiles of 128 tokens */
#define MOE_PLAN_KIND_COOPERATIVE 2 /* one cooperative kernel with two grid barriers */
#define MOE_PLAN_KIND_THREE 3       /* count, scan and rank kernels */

/*
 * moe_plan_create -- allocate a plan for up to `max_tokens` tokens of shape (k, E, R).
 * Allocates device memory once (cudaMalloc); later moe_plan calls reuse it.
 * On success *out receives the plan.  max_tokens >= 0.
 */
MOE_API moe_status moe_plan_create(int32_t max_tokens, int32_t k, int32_t E, int32_t R,
                           moe_plan_t *out);

/*
 * moe_plan_create_aligned -- as moe_plan_create, with every expert segment of the receive
 * buffer starting on a multiple of `align` rows (1 <= align <= 65536), e.g. the row tile of
 * a grouped GEMM over the experts.  The rows between an expert's last entry and the next
 * segment are padding: dispatch does not write them, combine does not read them, and
 * src_tok/src_j mark them -1.  Receive buffers then need N*k + E*(align-1) rows
 * (moe_plan_view.recv_rows).  The logical segments are the pages' (FUSCO summary,
 * Group 3); the alignment is this library's option for the consumer of the segments.
 */
MOE_API moe_status moe_plan_create_aligned(int32_t max_tokens, int32_t k, int32_t E, int32_t R,
                                           int32_t align, moe_plan_t *out);

/* Flags of moe_plan_create_ex. */
#define MOE_PLAN_NO_DEDUP_LISTS 1u  /* moe_plan skips the per-rank lists rtok / fanout */

/*
 * moe_plan_create_ex -- as moe_plan_create_aligned, with option flags.  With
 * MOE_PLAN_NO_DEDUP_LISTS the plan's per-rank dedup lists (rtok, fanout) are not written by
 * moe_plan (their contents are then undefined); everything else, rcnt and rtok_off
 * included, is.  Neither dispatch nor combine reads the lists, so callers that do not use
 * them save the planner their stores.  Unknown flags return MOE_EINVAL.
 */
MOE_API moe_status moe_plan_create_ex(int32_t max_tokens, int32_t k, int32_t E, int32_t R,
                                      int32_t align, uint32_t flags, moe_plan_t *out);

/*
 * moe_plan -- build the logical-segment plan of one routing (FUSCO abstract: the
 * "lightweight planning" that turns the captured layout into placements and drops
 * redundant transfers; DySHARP blog, section 5: a destination maps a token's logical
 * index to its own local address, which is what slot[] is).
 *
 *   topk_idx  device int32 [N, k]  expert ids of each token (caller-owned, read here)
 *   topk_w    device fp32  [N, k]  routing weights; only the pointer is kept, and
 *                                  moe_combine reads it, so it must stay valid and
 *                                  unchanged until the last combine using this plan
 *   N, k, E, R                     tokens, experts per token, experts, ranks
 *   stream                         cudaStream_t as void*
 *   plan      in/out: if *plan is NULL a plan sized for N tokens is created (device
 *             allocation); otherwise *plan is reused and must have been created with
 *             the same (k, E, R) and capacity >= N, else MOE_EINVAL.
 *
 * An id of -1 marks an entry the router dropped: it gets slot -1, no receive row and no
 * share of the combine, and it is not an error.
 *
 * Computes, for expert e on rank e / (E/R):
 *   cnt[e], expert_off = exclusive scan of cnt (each rounded up to the plan's alignment),
 *   rank_off[r] = expert_off[r*E/R];
 *   slot[t,j] = expert_off[e] + #{t' < t : e in topk_idx[t',:]} (stable, ascending t);
 *   src_tok/src_j = inverse of slot;
 *   rcnt[r] = #{t : some expert of t is on r}, rtok_off = exclusive scan of rcnt,
 *   rtok/fanout = the tokens of rank r in ascending order with the mask of their
 *   columns on r -- one move per (token, rank) pair.
 * Deterministic (no result depends on thread timing).  Enqueues one kernel: a single
 * block for N <= 128 (one tile); else one block per 128 tokens in thread-block clusters of
 * up to 16 blocks, which combine their counts through distributed shared memory and, with
 * more than one cluster, exchange the clusters' totals once through global memory (a
 * cooperative launch); where those clusters cannot all be resident, one cooperative kernel
 * with two grid barriers, or three kernels where even that grid cannot be co-resident.
 * A device wait that runs out sets MOE_ERR_TIMEOUT, which stays in the error word until
 * moe_plan_check reports it and rearms the plan.
 */
MOE_API moe_status moe_plan(const int32_t *topk_idx, const float *topk_w, int32_t N, int32_t k,
                    int32_t E, int32_t R, void *stream, moe_plan_t *plan);

/*
 * moe_dispatch -- recv[slot[t,j], :] = x[t, :] for every entry (FUSCO abstract and the
 * FUSCO summary, Group 3: rows are placed straight into the expert-major layout with no
 * intermediate buffer or later rearrangement).  Each token row is read from memory once
 * and written to all of its k receive rows.
 *
 *   x           device [N, H] of `dtype` (bf16, or fp8 e4m3 bytes)
 *   dtype       MOE_BF16 or MOE_FP8E4M3
 *   x_scale     device fp32 [N, H/128] for fp8 (moved with its row), NULL for bf16
 *   H           elements per row
 *   plan        a plan built by moe_plan (its N and k are used)
 *   recv        device [recv_rows, H] of `dtype`, caller-allocated (recv_rows = N*k for a
 *               tight plan); every row an entry maps to is written, others are untouched
 *   recv_scale  device fp32 [recv_rows, H/128] for fp8, NULL for bf16
 * Rows are copied bit for bit; nothing is converted.
 */
MOE_API moe_status moe_dispatch(const void *x, moe_dtype dtype, const float *x_scale, int32_t H,
                        moe_plan_t plan, void *recv, float *recv_scale, void *stream);

/*
 * moe_combine -- out[t, :] = bf16_rne( fp32 fma chain over j = 0..k-1 of
 * topk_w[t,j] * y[slot[t,j], :] ), starting from +0 (DySHARP blog, sections 1-2: the
 * experts' results for a token are brought back and summed).  The chain order is the
 * top-k column order, so the result does not depend on the launch configuration.
 *
 *   y     device bf16 [recv_rows, H]  expert outputs in the receive layout (rows no
 *         entry maps to are not read)
 *   H     elements per row (H % 8 == 0)
 *   plan  the plan whose slots laid out y; its weights pointer is read
 *   out   device bf16 [N, H], caller-allocated, fully overwritten
 */
MOE_API moe_status moe_combine(const void *y, int32_t H, moe_plan_t plan, void *out, void *stream);

/*
 * moe_plan_noalloc -- the plan of moe_plan, for callers that may not allocate device
 * memory: a process whose allocator owns every byte of the GPU, or a latency-critical
 * loop that cannot afford an allocation's device-wide synchronisation.  (The pages
 * describe no counterpart; this is a property of this library's interface.)
 *
 * Writes the same arrays, with the same values, as moe_plan into arrays the caller
 * owns: cnt[E], expert_off[E+1], rcnt[R], rank_off[R+1], rtok_off[R+1], slot[N*k],
 * src_tok[N*k], src_j[N*k], rtok and fanout [N*min(k,R)], err[1] (all device, 4-byte
 * aligned).  Calls no cudaMalloc or cudaFree.  Its per-tile scratch counts live in one
 * fixed 1 MiB array in device memory that every GPU loading the library keeps until the
 * process exits; a call needing more than (E + R + 1) * ceil(N / 128) <= 262144 scratch
 * words returns MOE_EINVAL.  The first call on each device does a one-time set-up (it
 * looks up that array's device address); make that first call before any stream capture
 * begins.  All calls share the array, so calls whose kernels could overlap on the GPU race
 * and must be ordered (one stream, or events).  topk_w is not taken: moe_combine needs a
 * plan from moe_plan.
 *
 * The call runs on the current device (ordinals 0..63; another ordinal returns MOE_EINVAL),
 * not on the device that owns the arrays: topk_idx and every output must be device memory
 * of the current device (or managed memory), else MOE_EINVAL before anything is enqueued.
 * The array's device address is looked up once per device and kept, so cudaDeviceReset
 * between calls is not supported.
 */
MOE_API moe_status moe_plan_noalloc(const int32_t *topk_idx, int32_t N, int32_t k, int32_t E,
                                    int32_t R, int32_t *cnt, int32_t *expert_off, int32_t *rcnt,
                                    int32_t *rank_off, int32_t *rtok_off, int32_t *slot,
                                    int32_t *src_tok, int32_t *src_j, int32_t *rtok,
                                    uint32_t *fanout, uint32_t *err, void *stream);

/*
 * moe_combine_ranked -- the combine with the reduction grouped by rank, the combine-side
 * counterpart of the per-rank dedup (DySHARP blog, section 2: the partial results that
 * several destinations produce for one token could be summed before travelling back;
 * section 5: a reducing load returns one result).  For each rank holding experts of token
 * t, in ascending rank order, a partial is formed as the fp32 fma chain over t's columns
 * on that rank (ascending column, from +0); the partials are added in fp32 in ascending
 * rank order (from +0) and the sum is rounded to bf16 (nearest even).  Arguments as for
 * moe_combine.  The result differs from moe_combine only by rounding order (within the
 * same error bound).  Uses the bulk-copy engine.
 */
MOE_API moe_status moe_combine_ranked(const void *y, int32_t H, moe_plan_t plan, void *out,
                                      void *stream);

/*
 * moe_dispatch_combine -- one dispatch and one combine in a single persistent launch, the
 * single-GPU form of DySHARP's token-centric kernel fusion (DySHARP blog, section 6:
 * Dispatch and Combine of different tokens run at the same time inside one kernel, each
 * token's work starting as soon as its inputs are ready).  The results are exactly those of
 *   moe_dispatch(x, dtype, x_scale, H_x, dispatch_plan, recv, recv_scale) and
 *   moe_combine(y, H_y, combine_plan, out)   (moe_combine_ranked when ranked != 0).
 * The two plans may differ (e.g. dispatch of micro-batch m+1 while micro-batch m combines).
 *
 * If y == recv (same plan, bf16, H_x == H_y), the combine reads the rows this call
 * dispatches: token t is combined only after its own rows have been written (per-token
 * ready flags in the plan; no other synchronisation is needed).  Otherwise y and recv must
 * not overlap (MOE_EINVAL).
 *
 * Calls moving less than MOE_TUNE_FUSED_MIN_KB of payload (320 MB by default; below it the
 * one-launch kernel's start-up outweighs the overlap) run the dispatch and combine kernels
 * one after the other on `stream` instead, with the same results.
 *
 * Arguments are those of moe_dispatch and moe_combine.  fp8 rows need H_x % 512 == 0 (scale
 * rows of a multiple of 16 bytes).  The launch is cooperative; calls that use the same
 * dispatch_plan must be ordered on the GPU (one stream, or events): the plan holds the
 * launch's work counters and flags.  A device wait that runs out (MOE_ERR_TIMEOUT in the
 * plans' error words) leaves the outputs incomplete; moe_plan_check then rearms the plan.
 */
MOE_API moe_status moe_dispatch_combine(const void *x, moe_dtype dtype, const float *x_scale,
                                        int32_t H_x, moe_plan_t dispatch_plan, void *recv,
                                        float *recv_scale, const void *y, int32_t H_y,
                                        moe_plan_t combine_plan, void *out, int32_t ranked,
                                        void *stream);

/*
 * moe_wait_selftest -- a diagnostic with no counterpart in the reference pages.  Runs one of
 * the library's bounded device waits on something that never completes and returns, in
 * *flags, the error word it leaves:
 *   which = 0  the per-token ready-flag wait of moe_dispatch_combine, on a flag nothing sets;
 *   which = 1  the mbarrier wait of the bulk-copy pipelines, on a barrier that expects two
 *              arrivals and gets one (no copy in flight);
 *   which = 2  the grid barrier of the cooperative plan kernel, in a grid of two blocks of
 *              which only one arrives;
 *   which = 3  the exchange wait of the group plan kernel, on two groups' arrival words of
 *              which only the first is ever set.
 * Each wait gives up after about one second; *flags is then MOE_ERR_TIMEOUT and the CUDA
 * context stays usable.  Synchronous: allocates three device words, launches two 32-thread
 * blocks on `stream`, waits for them and frees the words.  MOE_EINVAL for another `which`
 * or a NULL `flags`; MOE_ECUDA if a CUDA call fails.
 */
MOE_API moe_status moe_wait_selftest(int32_t which, void *stream, uint32_t *flags);

/* moe_plan_query -- fill *view with the plan's shape and device pointers. */
MOE_API moe_status moe_plan_query(moe_plan_t plan, moe_plan_view *view);

/*
 * moe_plan_check -- wait for `stream`, then copy the plan's error word to *flags
 * (MOE_ERR_* bits; 0 = the routing was valid and every wait finished).  After a reported
 * MOE_ERR_TIMEOUT it also rearms the plan: its grid-barrier and work words, its ready flags
 * and its error word.
 */
MOE_API moe_status moe_plan_check(moe_plan_t plan, void *stream, uint32_t *flags);

/* moe_plan_destroy -- free the plan (synchronises the device). NULL is a no-op. */
MOE_API moe_status moe_plan_destroy(moe_plan_t plan);

/* Message of the last failing call on this host thread ("" if none). */
MOE_API const char *moe_last_error(void);

/* Library version string. */
MOE_API const char *moe_version(void);

/* Launch parameters that moe_tune can override (process-wide; 0 restores the default).
 * They change speed only, never results.  Not safe to call while another host thread
 * is launching. */
typedef enum {
    MOE_TUNE_DISPATCH_STAGES = 0,        /* shared-memory row stages per dispatch warp (2..8) */
    MOE_TUNE_DISPATCH_LAG = 1,           /* store groups a warp keeps in flight (1..stages-1) */
    MOE_TUNE_DISPATCH_CTAS_PER_SM = 2,   /* cap on resident dispatch CTAs per SM */
    MOE_TUNE_DISPATCH_WARPS_PER_CTA = 3, /* dispatch warps per CTA (1..4) */
                                         /* 4: retired (an engine that was slower) */
    MOE_TUNE_COMBINE_CTAS_PER_SM = 5,    /* cap on resident combine CTAs per SM */
    MOE_TUNE_COMBINE_STAGES = 6,         /* bulk combine: shared-memory stages (2..16) */
                                         /* 7: retired */
    MOE_TUNE_COMBINE_SMEM_KB = 8,        /* bulk combine: shared-memory budget per CTA (KB) */
    MOE_TUNE_DISPATCH_UNITS_PER_WARP = 9, /* (token, chunk) units per dispatch warp */
    MOE_TUNE_COMBINE_TOKENS_PER_CTA = 10, /* tokens per bulk-combine CTA (0: runs of about
                                            256 KB of rows for k > 4, 8 tokens for k <= 4,
                                            resized to fill whole waves of resident CTAs
                                            when there are fewer than three) */
    MOE_TUNE_PLAN_ENGINE = 11,           /* 0 or 1: automatic, 2: three kernels, 3: no cluster
                                            kernel (the cooperative one for N > 128) */
    MOE_TUNE_FUSED_CTAS_PER_SM = 12,     /* moe_dispatch_combine: resident CTAs per SM */
    MOE_TUNE_FUSED_DISPATCH_SHARE = 13,  /* moe_dispatch_combine: % of CTAs that start on dispatch */
    MOE_TUNE_FUSED_DISPATCH_RUN = 14,    /* moe_dispatch_combine: tokens per dispatch work item
                                            (1..32; 0: about 64 KB of traffic, 144 KB when
                                            the combine waits on ready flags) */
    MOE_TUNE_FUSED_COMBINE_RUN = 15,     /* moe_dispatch_combine: tokens per combine work item */
    MOE_TUNE_FUSED_SMEM_KB = 16,         /* moe_dispatch_combine: shared memory per CTA (KB) */
    MOE_TUNE_FUSED_MIN_KB = 17,          /* moe_dispatch_combine: least traffic (KB) for the
                                            one-launch kernel; smaller calls run the two
                                            kernels back to back (default 327680 = 320 MB) */
    MOE_TUNE_COMBINE_MAX_CW = 18,        /* bulk combine: most consumer warps per CTA (4 or 8;
                                            default 8: k <= 4 uses 8, wider k uses 4 or fewer) */
    MOE_TUNE_PLAN_CLUSTER = 19,          /* plan: most 128-token tiles per thread-block cluster
                                            (1..16; default 16) */
    MOE_TUNE_PDL = 20,                   /* 0 or 1: kernels are programmatic dependent launches
                                            (each may start while the previous kernel on the
                                            stream finishes), 2: ordinary launches */
    MOE_TUNE_PLAN_MATCH = 21,            /* plan: how a token's ids are compared: 0 by k (match
                                            instructions for k > 16), 1 shuffle compares,
                                            2 warp match instructions */
    MOE_TUNE_DISPATCH_SPLIT_UNITS = 22,  /* dispatch: below this many (token, chunk) units rows
                                            are cut into chunks of >= 2 KB (0: 4 per SM;
                                            1: never) */
    MOE_TUNE_COMBINE_SPLIT = 23          /* combine: CTAs that share a run of tokens when the
                                            tokens are few (0: automatic; 1: never) */
} moe_knob;

MOE_API moe_status moe_tune(moe_knob knob, int32_t value);

#ifdef __cplusplus
}
#endif

#endif /* MOE_SHUFFLE_H */
