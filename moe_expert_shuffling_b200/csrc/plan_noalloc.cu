// moe_plan_noalloc: the planner for callers that may not allocate device memory.
//
// Some callers cannot call cudaMalloc: a serving process or framework that reserves all
// of the GPU's memory up front through its own allocator and does not let a library
// take memory behind its back, or a latency-critical loop where an allocation (which
// can synchronise the whole device) is not acceptable.  For them this entry point
// writes the plan into arrays the caller owns and keeps its per-tile scratch counts in
// a fixed array in device memory that the library declares once (kScratchWords words,
// 1 MiB).  Every GPU that loads the library holds that array until the process exits.
//
// All calls share the array.  It keeps whatever the last call left in it; nothing in it
// has to start at zero, because each call writes every scratch word it later reads.
// Calls whose kernels overlap on the GPU (for example on two streams without an
// ordering between them) race on the array and must not be issued.
//
// The array's device address is looked up once per device ordinal (below 64) and kept, so
// the library does not support cudaDeviceReset between calls: a new context would be given
// the old context's address.
#include <mutex>

#include "common.cuh"
#include "internal.cuh"

namespace {

constexpr int64_t kScratchWords = 262144;  // 1 MiB of int32 scratch

__device__ __align__(256) int32_t g_plan_scratch[kScratchWords];

// Device address of g_plan_scratch per device (host code only sees a stand-in for the
// symbol, so the address must come from cudaGetSymbolAddress with the device current).
struct ScratchSlot {
    bool ready = false;
    int32_t *ptr = nullptr;
};
ScratchSlot g_scratch[64];
std::mutex g_scratch_mu;

moe_status scratch_address(int dev, int32_t **out)
{
    if (dev < 0 || dev >= 64)
        return moe::record_error(MOE_EINVAL, "device %d is outside the supported range", dev);
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch[dev].ready) {
        void *p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_plan_scratch);
        if (e != cudaSuccess)
            return moe::record_error(MOE_ECUDA, "cudaGetSymbolAddress(scratch): %s (%s)",
                                     cudaGetErrorName(e), cudaGetErrorString(e));
        g_scratch[dev].ptr = static_cast<int32_t *>(p);
        g_scratch[dev].ready = true;
    }
    *out = g_scratch[dev].ptr;
    return MOE_OK;
}

bool aligned4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

// The caller owns every array, so a host pointer or another GPU's pointer would reach the
// kernels unchecked; reject anything but device memory of `dev` (or managed memory) here.
moe_status check_device_array(const void *p, int dev, const char *name)
{
    cudaPointerAttributes a{};
    const cudaError_t e = cudaPointerGetAttributes(&a, p);
    if (e != cudaSuccess) {
        (void)cudaGetLastError();
        return moe::record_error(MOE_EINVAL, "moe_plan_noalloc: %s is not device memory (%s)",
                                 name, cudaGetErrorString(e));
    }
    if (a.type == cudaMemoryTypeManaged)
        return MOE_OK;
    if (a.type != cudaMemoryTypeDevice)
        return moe::record_error(MOE_EINVAL,
                                 "moe_plan_noalloc: %s is host memory, not device memory", name);
    if (a.device != dev)
        return moe::record_error(MOE_EINVAL,
                                 "moe_plan_noalloc: %s lives on device %d but device %d is current",
                                 name, a.device, dev);
    return MOE_OK;
}

}  // namespace

extern "C" moe_status moe_plan_noalloc(const int32_t *topk_idx, int32_t N, int32_t k, int32_t E,
                                       int32_t R, int32_t *cnt, int32_t *expert_off,
                                       int32_t *rcnt, int32_t *rank_off, int32_t *rtok_off,
                                       int32_t *slot, int32_t *src_tok, int32_t *src_j,
                                       int32_t *rtok, uint32_t *fanout, uint32_t *err,
                                       void *stream)
{
    if (N < 0)
        return moe::record_error(MOE_EINVAL, "N must be >= 0 (got %d)", N);
    if (k < 1 || k > moe::kMaxTopk)
        return moe::record_error(MOE_EINVAL, "k must be in [1, %d] (got %d)", moe::kMaxTopk, k);
    if (E < k || E > moe::kMaxExperts)
        return moe::record_error(MOE_EINVAL, "E must be in [k, %d] (got E=%d, k=%d)",
                                 moe::kMaxExperts, E, k);
    if (R < 1 || E % R != 0)
        return moe::record_error(MOE_EINVAL, "R must divide E (got E=%d, R=%d)", E, R);
    if (static_cast<int64_t>(N) * k >= (int64_t(1) << 31))
        return moe::record_error(MOE_EINVAL, "N*k must be < 2^31");
    const int64_t tiles = moe::ceil_div(N, moe::kPlanTile);
    const int64_t need = (static_cast<int64_t>(E) + R + 1) * (tiles > 0 ? tiles : 1);
    if (need > kScratchWords)
        return moe::record_error(
            MOE_EINVAL,
            "moe_plan_noalloc: N=%d with E=%d, R=%d needs %lld scratch words, the fixed "
            "array holds %lld; use fewer tokens per call or moe_plan",
            N, E, R, static_cast<long long>(need), static_cast<long long>(kScratchWords));
    if (!cnt || !expert_off || !rcnt || !rank_off || !rtok_off || !err)
        return moe::record_error(MOE_EINVAL, "every output array must be given");
    if (N > 0 && (!topk_idx || !slot || !src_tok || !src_j || !rtok || !fanout))
        return moe::record_error(MOE_EINVAL, "topk_idx and the per-entry outputs must be given");
    const void *ptrs[] = {topk_idx, cnt, expert_off, rcnt, rank_off, rtok_off, slot,
                          src_tok, src_j, rtok, fanout, err};
    for (const void *q : ptrs)
        if (!aligned4(q))
            return moe::record_error(MOE_EINVAL, "arrays must be 4-byte aligned");

    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return moe::record_error(MOE_ECUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    const char *names[] = {"topk_idx", "cnt", "expert_off", "rcnt", "rank_off", "rtok_off", "slot",
                           "src_tok", "src_j", "rtok", "fanout", "err"};
    for (int i = 0; i < 12; ++i) {
        if (!ptrs[i])
            continue;  // only the per-entry arrays may be NULL, and only when N == 0
        const moe_status pst = check_device_array(ptrs[i], dev, names[i]);
        if (pst != MOE_OK)
            return pst;
    }
    int32_t *scratch = nullptr;
    const moe_status st = scratch_address(dev, &scratch);
    if (st != MOE_OK)
        return st;

    const int64_t t = tiles > 0 ? tiles : 1;
    moe::PlanArrays a;
    a.topk_idx = topk_idx;
    a.N = N;
    a.k = k;
    a.E = E;
    a.R = R;
    a.rtok_cap = static_cast<int64_t>(N) * (k < R ? k : R);
    a.cnt = cnt;
    a.expert_off = expert_off;
    a.rcnt = rcnt;
    a.rank_off = rank_off;
    a.rtok_off = rtok_off;
    a.slot = slot;
    a.src_tok = src_tok;
    a.src_j = src_j;
    a.rtok = rtok;
    a.fanout = fanout;
    a.err = err;
    a.tile_cnt = scratch;
    a.tile_rcnt = scratch + static_cast<int64_t>(E) * t;
    a.tile_err = reinterpret_cast<uint32_t *>(scratch + static_cast<int64_t>(E + R) * t);
    e = moe::launch_plan_arrays(a, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess)
        return moe::record_error(MOE_ECUDA, "plan kernels: %s (%s)", cudaGetErrorName(e),
                                 cudaGetErrorString(e));
    moe::record_error(MOE_OK, "");
    return MOE_OK;
}
