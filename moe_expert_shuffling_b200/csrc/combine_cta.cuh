// The combine CTA's producer and consumer loops, shared by the combine kernel and the
// fused dispatch-and-combine kernel.
//
// out[t] = bf16_rne( fp32 fma chain over j = 0..k-1 of w[t, j] * y[slot[t, j]] ), from +0
// (DySHARP blog, sections 1-2: the expert results of a token are brought back and summed).
// A CTA is one producer warp and CW consumer warps.  A unit is (token, CW * 512-byte
// column chunk of every row).  The producer issues one bulk async copy per routed row
// chunk (lane j copies row slot[t, j]) into a ring stage that completes on a "full"
// mbarrier; each consumer thread reduces 8 columns over the k rows from shared memory,
// writes 16 bytes of out and releases the stage on its "empty" mbarrier.
//
// Rank-grouped order (RANKED): per rank (ascending) an fp32 fma chain over the token's
// columns on that rank (ascending), and the partials added in ascending rank order.  The
// producer puts the token's kept rows into the stage already sorted by (rank, column), so
// consumers read rows at fixed offsets and carry only the sorted weights and a bitmask of
// the positions where a new rank starts.
#pragma once

#include <cuda_bf16.h>

#include "common.cuh"

namespace moe {

__device__ __forceinline__ void fma_bf16x8(float *acc, float wj, const uint4 &v)
{
    const uint32_t words[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const float lo = __uint_as_float(words[q] << 16);
        const float hi = __uint_as_float(words[q] & 0xffff0000u);
        acc[2 * q] = __fmaf_rn(wj, lo, acc[2 * q]);
        acc[2 * q + 1] = __fmaf_rn(wj, hi, acc[2 * q + 1]);
    }
}

__device__ __forceinline__ uint4 pack_bf16x8(const float *acc)
{
    uint32_t words[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(acc[2 * q], acc[2 * q + 1]);
        words[q] = *reinterpret_cast<const uint32_t *>(&h);
    }
    return make_uint4(words[0], words[1], words[2], words[3]);
}

// A unit covers CW * 512 bytes of each of the token's k rows: one 16-byte vector per
// consumer thread, CW consumer warps.  The chunk narrows as k grows so that a stage
// (k x chunk) stays at 16 KB or less: CW = 8 for k <= 4, 4 for k <= 8, 2 for k <= 16,
// 1 for k <= 32.
template <int CW>
struct Shape {
    static constexpr uint32_t kChunk = 512u * CW;
    static constexpr int kThreads = 32 * (1 + CW);
};
constexpr int kMaxBulkStages = 16;
constexpr int32_t kNoRank = 0x7fffffff;

struct CombineBulkParams {
    const uint8_t *y;
    const int32_t *slot;
    const float *w;
    uint8_t *out;
    uint32_t *err;
    int32_t N, k, n_rows;
    uint32_t row_bytes, nchunks, stages, stage_bytes, bar_bytes;
    uint32_t per_cta;       // tokens of each CTA: [cta * per_cta, +per_cta)
    const int32_t *rank_off;  // [R+1] first receive row of each rank (rank-grouped order)
    int32_t R;
    uint32_t ring_bytes;    // bytes of the stage ring (the rank tables follow it)
    uint32_t csplit;        // CTAs sharing one run of tokens, each taking a range of chunks
};

// Shared-memory layout of one combine CTA: 2S mbarriers, the ring, then (rank-grouped
// order) the rank offsets and 64 words per consumer warp.
struct CombineRing {
    uint64_t *full, *empty;
    uint8_t *ring;
    int32_t *roff_s;
    float *wo_s;    // this consumer warp's weights in (rank, column) order
    int32_t *ro_s;  // and their ranks
    int S;

    template <bool RANKED>
    __device__ __forceinline__ void carve(const CombineBulkParams &p, uint8_t *smem, int warp)
    {
        S = static_cast<int>(p.stages);
        full = reinterpret_cast<uint64_t *>(smem);
        empty = full + S;
        ring = smem + p.bar_bytes;
        roff_s = reinterpret_cast<int32_t *>(ring + p.ring_bytes);
        wo_s = reinterpret_cast<float *>(roff_s + (RANKED ? p.R + 1 : 0) +
                                         (warp > 0 ? (warp - 1) * 64 : 0));
        ro_s = reinterpret_cast<int32_t *>(wo_s + 32);
    }

    // thread 0 only; a __syncthreads must follow before any use
    template <int CW>
    __device__ __forceinline__ void init() const
    {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], CW);
        }
        mbar_init_fence();
    }
};

// Rank of receive row s: the r with roff[r] <= s < roff[r + 1] (rows are grouped by rank).
__device__ __forceinline__ int32_t rank_of_row(const int32_t *roff, int R, int32_t s)
{
    int lo = 0, hi = R;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (roff[mid] <= s)
            lo = mid;
        else
            hi = mid;
    }
    return lo;
}

// Position of this lane's column in the token's (rank, column) order, lanes j < k holding
// column j with rank rj (kNoRank for a dropped column, which sorts after every kept one).
__device__ __forceinline__ int rank_order_pos(int32_t rj, int k, int lane)
{
    int pos = 0;
    for (int q = 0; q < k; ++q) {
        const int32_t rq = __shfl_sync(0xffffffffu, rj, q);
        pos += (rq < rj || (rq == rj && q < lane)) ? 1 : 0;
    }
    return pos;
}

// Wait (one thread) until flag == epoch; false after the wait limit, or as soon as another
// CTA has reported a timeout in *err.
__device__ __forceinline__ bool wait_flag(const uint32_t *flag, uint32_t epoch, const uint32_t *err)
{
    if (ld_acquire_gpu(flag) == epoch)
        return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 1; it < (1u << 30); ++it) {
        __nanosleep(64);
        if (ld_acquire_gpu(flag) == epoch)
            return true;
        if ((it & 15u) == 0 &&
            (global_timer_ns() - t0 > kWaitLimitNs || (ld_relaxed_gpu(err) & MOE_ERR_TIMEOUT)))
            return false;
    }
    return false;
}

// Producer warp over tokens [b, b + n_tok), chunks [c_lo, c_hi) of each.  `i` is the ring
// position (chunks issued so far), carried across runs.  `s_cur` holds lane j's slot of token b (j < k) or -1.  With
// `ready`, token t's rows are read only once ready[t] == epoch (they are being written by
// the same launch).  Returns false after a timeout (MOE_ERR_TIMEOUT set).
template <int KMAX, int CW, bool RANKED>
__device__ __forceinline__ bool combine_produce(const CombineBulkParams &p, const CombineRing &r,
                                                uint32_t b, int n_tok, int32_t s_cur, int &i,
                                                const uint32_t *ready, uint32_t epoch,
                                                uint32_t c_lo = 0u, uint32_t c_hi = ~0u)
{
    c_hi = min(c_hi, p.nchunks);
    constexpr uint32_t kChunk_ = Shape<CW>::kChunk;
    const int lane = threadIdx.x & 31;
    const int k = p.k;
    const int S = r.S;
    bool ok = true;
    for (int m = 0; m < n_tok && ok; ++m) {
        const uint32_t t = b + static_cast<uint32_t>(m);
        int32_t s_nxt = -1;
        if (m + 1 < n_tok && lane < k)
            s_nxt = __ldg(p.slot + static_cast<int64_t>(t + 1) * k + lane);
        const bool valid =
            lane < k && static_cast<uint32_t>(s_cur) < static_cast<uint32_t>(p.n_rows);
        const uint32_t nv = __popc(__ballot_sync(0xffffffffu, valid));
        uint32_t dst = static_cast<uint32_t>(lane) * kChunk_;
        if (RANKED)
            dst = static_cast<uint32_t>(rank_order_pos(
                      valid ? rank_of_row(r.roff_s, p.R, s_cur) : kNoRank, k, lane)) *
                  kChunk_;
        if (ready != nullptr) {
            bool rdy = true;
            if (lane == 0)
                rdy = wait_flag(ready + t, epoch, p.err);
            if (!__shfl_sync(0xffffffffu, rdy, 0)) {
                ok = false;
                break;
            }
            if (valid) {
                (void)ld_acquire_gpu(ready + t);
                fence_proxy_async_global();
            }
        }
        for (uint32_t c = c_lo; c < c_hi; ++c, ++i) {
            const int st = i % S;
            const uint32_t ph = static_cast<uint32_t>((i / S) & 1);
            if (!__all_sync(0xffffffffu, mbar_wait_bounded(&r.empty[st], ph ^ 1u))) {
                ok = false;
                break;
            }
            const uint32_t off = c * kChunk_;
            const uint32_t len = min(kChunk_, p.row_bytes - off);
            if (lane == 0)
                mbar_arrive_expect_tx(&r.full[st], nv * len);
            __syncwarp();
            if (valid)
                bulk_load(r.ring + static_cast<size_t>(st) * p.stage_bytes + dst,
                          p.y + static_cast<int64_t>(s_cur) * p.row_bytes + off, len,
                          &r.full[st]);
        }
        s_cur = s_nxt;
    }
    if (!ok) {
        if (lane == 0)
            atomicOr(p.err, MOE_ERR_TIMEOUT);
        // let the copies of the last stages land before the ring is reused or released
        for (int q = (i > S ? i - S : 0); q < i; ++q)
            (void)mbar_wait_bounded(&r.full[q % S], static_cast<uint32_t>((q / S) & 1));
    }
    return ok;
}

// Consumer warps over tokens [b, b + n_tok), chunks [c_lo, c_hi) of each: thread v owns bytes
// [16v, 16v + 16) of every chunk.  A token's valid columns (bitmask) and weights are broadcast once per token and
// kept in registers; each chunk then costs k shared loads, 8k fmas and one 16-byte store.
// `s_nxt` / `w_nxt` hold lane j's slot and weight of token b.  Returns false after a
// timeout (MOE_ERR_TIMEOUT set).
template <int KMAX, int CW, bool RANKED>
__device__ __forceinline__ bool combine_consume(const CombineBulkParams &p, const CombineRing &r,
                                                uint32_t b, int n_tok, int32_t s_nxt,
                                                float w_nxt, int &i, uint32_t c_lo = 0u,
                                                uint32_t c_hi = ~0u)
{
    c_hi = min(c_hi, p.nchunks);
    constexpr uint32_t kChunk_ = Shape<CW>::kChunk;
    constexpr int kJ = KMAX < 8 ? KMAX : 8;  // rows held in registers at once
    const int lane = threadIdx.x & 31;
    const int k = p.k;
    const int S = r.S;
    const uint32_t v16 = static_cast<uint32_t>(threadIdx.x - 32) * 16u;
    for (int m = 0; m < n_tok; ++m) {
        const uint32_t t = b + static_cast<uint32_t>(m);
        const uint32_t vmask = __ballot_sync(
            0xffffffffu,
            lane < k && static_cast<uint32_t>(s_nxt) < static_cast<uint32_t>(p.n_rows));
        float wv[KMAX];
        uint32_t nv = 0, starts = 0;  // ranked: kept columns; positions opening a new rank
        if (!RANKED) {
#pragma unroll
            for (int j = 0; j < KMAX; ++j)
                wv[j] = __shfl_sync(0xffffffffu, w_nxt, j);
        } else {
            nv = __popc(vmask);
            const int32_t rj =
                ((vmask >> lane) & 1u) ? rank_of_row(r.roff_s, p.R, s_nxt) : kNoRank;
            const int pos = rank_order_pos(rj, k, lane);
            __syncwarp();
            if (lane < k) {
                r.wo_s[pos] = w_nxt;
                r.ro_s[pos] = rj;
            }
            __syncwarp();
            const float w_sorted = lane < k ? r.wo_s[lane] : 0.f;
            const int32_t r_sorted = lane < k ? r.ro_s[lane] : kNoRank;
            const int32_t r_before = __shfl_up_sync(0xffffffffu, r_sorted, 1);
            starts = __ballot_sync(0xffffffffu, lane > 0 && static_cast<uint32_t>(lane) < nv &&
                                                    r_sorted != r_before);
#pragma unroll
            for (int j = 0; j < KMAX; ++j)
                wv[j] = __shfl_sync(0xffffffffu, w_sorted, j);
        }
        if (m + 1 < n_tok && lane < k) {
            s_nxt = __ldg(p.slot + static_cast<int64_t>(t + 1) * k + lane);
            w_nxt = __ldg(p.w + static_cast<int64_t>(t + 1) * k + lane);
        }
        for (uint32_t c = c_lo; c < c_hi; ++c, ++i) {
            const int st = i % S;
            const uint32_t ph = static_cast<uint32_t>((i / S) & 1);
            if (!__all_sync(0xffffffffu, mbar_wait_bounded(&r.full[st], ph))) {
                if (lane == 0)
                    atomicOr(p.err, MOE_ERR_TIMEOUT);
                return false;
            }
            const uint32_t off = c * kChunk_;
            const uint32_t len = min(kChunk_, p.row_bytes - off);
            const uint8_t *stage = r.ring + static_cast<size_t>(st) * p.stage_bytes + v16;
            const bool mine = v16 < len;
            float acc[8], part[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                acc[e] = 0.f;
                part[e] = 0.f;
            }
#pragma unroll
            for (int j0 = 0; j0 < KMAX; j0 += kJ) {
                if (j0 >= k)
                    break;  // warp-uniform
                uint4 q[kJ];
#pragma unroll
                for (int jj = 0; jj < kJ; ++jj) {
                    const int j = j0 + jj;
                    const bool kept = RANKED ? static_cast<uint32_t>(j) < nv : ((vmask >> j) & 1u);
                    q[jj] = (mine && kept) ? lds_v4(stage + j * kChunk_)
                                           : make_uint4(0u, 0u, 0u, 0u);
                }
                if (j0 + kJ >= k) {
                    // every row of this stage is in registers: release it to the producer
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive(&r.empty[st]);
                }
#pragma unroll
                for (int jj = 0; jj < kJ; ++jj) {
                    const int j = j0 + jj;
                    if (RANKED) {
                        if (static_cast<uint32_t>(j) >= nv)
                            continue;
                        if ((starts >> j) & 1u) {
                            // close the previous rank's chain
#pragma unroll
                            for (int e = 0; e < 8; ++e) {
                                acc[e] = __fadd_rn(acc[e], part[e]);
                                part[e] = 0.f;
                            }
                        }
                        fma_bf16x8(part, wv[j], q[jj]);
                    } else if ((vmask >> j) & 1u) {
                        fma_bf16x8(acc, wv[j], q[jj]);
                    }
                }
            }
            if (RANKED && nv > 0) {
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    acc[e] = __fadd_rn(acc[e], part[e]);
            }
            if (mine)
                st_stream_v4(p.out + static_cast<int64_t>(t) * p.row_bytes + off + v16,
                             pack_bf16x8(acc));
        }
    }
    return true;
}

}  // namespace moe
