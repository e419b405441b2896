// C ABI of libmoeshuffle: argument checks, plan ownership and kernel launches.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>
#include <string>

#include "common.cuh"
#include "internal.cuh"

namespace {

thread_local std::string g_last_error;

moe_status fail(moe_status st, const char *fmt, ...)
{
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return st;
}

moe_status ok()
{
    g_last_error.clear();
    return MOE_OK;
}

moe_status cuda_fail(cudaError_t e, const char *what)
{
    return fail(MOE_ECUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

moe_status check_shape(int64_t N, int32_t k, int32_t E, int32_t R)
{
    if (N < 0)
        return fail(MOE_EINVAL, "N must be >= 0 (got %lld)", static_cast<long long>(N));
    if (k < 1 || k > moe::kMaxTopk)
        return fail(MOE_EINVAL, "k must be in [1, %d] (got %d)", moe::kMaxTopk, k);
    if (E < k || E > moe::kMaxExperts)
        return fail(MOE_EINVAL, "E must be in [k, %d] (got E=%d, k=%d)", moe::kMaxExperts, E, k);
    if (R < 1 || E % R != 0)
        return fail(MOE_EINVAL, "R must divide E (got E=%d, R=%d)", E, R);
    if (N * k >= (int64_t(1) << 31))
        return fail(MOE_EINVAL, "N*k must be < 2^31 (got %lld)", static_cast<long long>(N * k));
    return MOE_OK;
}

moe_status current_device(int *dev)
{
    cudaError_t e = cudaGetDevice(dev);
    if (e != cudaSuccess)
        return cuda_fail(e, "cudaGetDevice");
    return MOE_OK;
}

moe_status check_plan_device(const moe_plan_s *p)
{
    int dev = 0;
    moe_status st = current_device(&dev);
    if (st != MOE_OK)
        return st;
    if (dev != p->device)
        return fail(MOE_EINVAL, "plan lives on device %d but device %d is current", p->device,
                    dev);
    return MOE_OK;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

namespace moe {

moe_status record_error(moe_status st, const char *fmt, ...)
{
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return st;
}

Tuning &tuning()
{
    static Tuning t;
    return t;
}

int sm_count(int device)
{
    static int cache[64] = {0};
    if (device < 0 || device >= 64)
        return 148;
    if (cache[device] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, device) != cudaSuccess ||
            n <= 0)
            n = 148;
        cache[device] = n;
    }
    return cache[device];
}

int max_smem_optin(int device)
{
    static int cache[64] = {0};
    if (device < 0 || device >= 64)
        return 0;
    if (cache[device] == 0) {
        int v = 0;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, device) !=
                cudaSuccess ||
            v <= 0)
            v = 48 * 1024;
        cache[device] = v;
    }
    return cache[device];
}

cudaError_t launch_ex(const void *kernel, void **args, dim3 grid, dim3 block, size_t smem,
                      cudaStream_t stream, bool cooperative, int device,
                      const cudaLaunchAttribute *extra, int n_extra)
{
    // [device][cooperative]: 1 once a programmatic launch of that kind succeeded, -1 once
    // the runtime refused the attribute for it
    static int pdl_state[64][2] = {};
    const int dv = device >= 0 && device < 64 ? device : 0;
    const int kind = cooperative ? 1 : 0;
    bool pdl = tuning().pdl != 2 && pdl_state[dv][kind] >= 0;
    if (pdl && pdl_state[dv][kind] == 0) {
        // the first launch of a kind is not tried inside a stream capture, where a refused
        // launch would invalidate the capture
        cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
        if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) {
            (void)cudaGetLastError();
            pdl = false;
        } else if (cs != cudaStreamCaptureStatusNone) {
            pdl = false;
        }
    }
    cudaLaunchAttribute attr[4];
    int n = 0;
    for (int i = 0; i < n_extra && n < 2; ++i)
        attr[n++] = extra[i];
    if (cooperative) {
        attr[n].id = cudaLaunchAttributeCooperative;
        attr[n].val.cooperative = 1;
        ++n;
    }
    const int without_pdl = n;
    if (pdl) {
        attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[n].val.programmaticStreamSerializationAllowed = 1;
        ++n;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = static_cast<unsigned>(n);
    cudaError_t e = cudaLaunchKernelExC(&cfg, kernel, args);
    if (pdl && e == cudaSuccess) {
        pdl_state[dv][kind] = 1;
    } else if (pdl && pdl_state[dv][kind] == 0) {
        (void)cudaGetLastError();
        cfg.numAttrs = static_cast<unsigned>(without_pdl);
        e = cudaLaunchKernelExC(&cfg, kernel, args);
        if (e == cudaSuccess)
            pdl_state[dv][kind] = -1;
    }
    return e;
}

namespace {
struct FitEntry {
    const void *kernel;
    int device, threads;
    size_t smem;
    int per_sm;
};
struct LimitEntry {
    const void *kernel;
    int device;
    size_t smem;
};
std::mutex g_fit_mu;
FitEntry g_fit[128];
int g_fit_n = 0;
LimitEntry g_limit[64];
int g_limit_n = 0;
}  // namespace

cudaError_t kernel_fit(const void *kernel, int device, int threads, size_t smem, int *per_sm)
{
    std::lock_guard<std::mutex> lock(g_fit_mu);
    for (int i = 0; i < g_fit_n; ++i) {
        const FitEntry &f = g_fit[i];
        if (f.kernel == kernel && f.device == device && f.threads == threads && f.smem == smem) {
            *per_sm = f.per_sm;
            return cudaSuccess;
        }
    }
    // raise the kernel's dynamic-shared-memory limit if this size needs more
    int li = -1;
    for (int i = 0; i < g_limit_n; ++i)
        if (g_limit[i].kernel == kernel && g_limit[i].device == device)
            li = i;
    if (smem > 48 * 1024 && (li < 0 || g_limit[li].smem < smem)) {
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem));
        if (e != cudaSuccess)
            return e;
        if (li < 0 && g_limit_n < 64)
            li = g_limit_n++;
        if (li >= 0)
            g_limit[li] = LimitEntry{kernel, device, smem};
    }
    int n = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, smem);
    if (e != cudaSuccess)
        return e;
    if (g_fit_n < 128)
        g_fit[g_fit_n++] = FitEntry{kernel, device, threads, smem, n};
    *per_sm = n;
    return cudaSuccess;
}

}  // namespace moe

extern "C" {

const char *moe_last_error(void) { return g_last_error.c_str(); }

const char *moe_version(void) { return "moeshuffle 0.2.0 (sm_100a)"; }

moe_status moe_tune(moe_knob knob, int32_t value)
{
    if (value < 0)
        return fail(MOE_EINVAL, "tuning values must be >= 0");
    moe::Tuning &t = moe::tuning();
    switch (knob) {
    case MOE_TUNE_DISPATCH_STAGES: t.dispatch_stages = value; break;
    case MOE_TUNE_DISPATCH_LAG: t.dispatch_lag = value; break;
    case MOE_TUNE_DISPATCH_CTAS_PER_SM: t.dispatch_ctas_per_sm = value; break;
    case MOE_TUNE_DISPATCH_WARPS_PER_CTA: t.dispatch_warps_per_cta = value; break;
    case MOE_TUNE_COMBINE_CTAS_PER_SM: t.combine_ctas_per_sm = value; break;
    case MOE_TUNE_COMBINE_STAGES: t.combine_stages = value; break;
    case MOE_TUNE_COMBINE_SMEM_KB: t.combine_smem_kb = value; break;
    case MOE_TUNE_DISPATCH_UNITS_PER_WARP: t.dispatch_units_per_warp = value; break;
    case MOE_TUNE_COMBINE_TOKENS_PER_CTA: t.combine_tokens_per_cta = value; break;
    case MOE_TUNE_PLAN_ENGINE: t.plan_engine = value; break;
    case MOE_TUNE_FUSED_CTAS_PER_SM: t.fused_ctas_per_sm = value; break;
    case MOE_TUNE_FUSED_DISPATCH_SHARE: t.fused_dispatch_share = value; break;
    case MOE_TUNE_FUSED_DISPATCH_RUN: t.fused_dispatch_run = value; break;
    case MOE_TUNE_FUSED_COMBINE_RUN: t.fused_combine_run = value; break;
    case MOE_TUNE_FUSED_SMEM_KB: t.fused_smem_kb = value; break;
    case MOE_TUNE_FUSED_MIN_KB: t.fused_min_kb = value; break;
    case MOE_TUNE_COMBINE_MAX_CW: t.combine_max_cw = value; break;
    case MOE_TUNE_PLAN_CLUSTER: t.plan_cluster = value; break;
    case MOE_TUNE_PDL: t.pdl = value; break;
    case MOE_TUNE_PLAN_MATCH: t.plan_match = value; break;
    case MOE_TUNE_DISPATCH_SPLIT_UNITS: t.dispatch_split_units = value; break;
    case MOE_TUNE_COMBINE_SPLIT: t.combine_split = value; break;
    default: return fail(MOE_EINVAL, "unknown tuning knob %d", static_cast<int>(knob));
    }
    return ok();
}

moe_status moe_plan_create(int32_t max_tokens, int32_t k, int32_t E, int32_t R, moe_plan_t *out)
{
    return moe_plan_create_aligned(max_tokens, k, E, R, 1, out);
}

moe_status moe_plan_create_aligned(int32_t max_tokens, int32_t k, int32_t E, int32_t R,
                                   int32_t align, moe_plan_t *out)
{
    return moe_plan_create_ex(max_tokens, k, E, R, align, 0u, out);
}

moe_status moe_plan_create_ex(int32_t max_tokens, int32_t k, int32_t E, int32_t R, int32_t align,
                              uint32_t flags, moe_plan_t *out)
{
    if (flags & ~static_cast<uint32_t>(MOE_PLAN_NO_DEDUP_LISTS))
        return fail(MOE_EINVAL, "unknown plan flags 0x%x", flags);
    if (!out)
        return fail(MOE_EINVAL, "out must not be NULL");
    *out = nullptr;
    moe_status st = check_shape(max_tokens, k, E, R);
    if (st != MOE_OK)
        return st;
    if (align < 1 || align > (1 << 16))
        return fail(MOE_EINVAL, "align must be in [1, 65536] (got %d)", align);
    if (moe::recv_rows(max_tokens, k, E, align) >= (int64_t(1) << 31))
        return fail(MOE_EINVAL, "N*k + E*(align-1) must be < 2^31");
    int dev = 0;
    if ((st = current_device(&dev)) != MOE_OK)
        return st;

    moe_plan_s *p = new (std::nothrow) moe_plan_s();
    if (!p)
        return fail(MOE_ENOMEM, "host allocation failed");
    p->cap = max_tokens;
    p->k = k;
    p->E = E;
    p->R = R;
    p->epr = E / R;
    p->device = dev;
    p->nt_cap = static_cast<int32_t>(moe::ceil_div(max_tokens, moe::kPlanTile));
    p->rtok_cap = static_cast<int64_t>(max_tokens) * (k < R ? k : R);
    p->align = align;
    p->rows_cap = moe::recv_rows(max_tokens, k, E, align);
    p->dedup_lists = (flags & MOE_PLAN_NO_DEDUP_LISTS) == 0;
    const int64_t rows = static_cast<int64_t>(max_tokens) * k;
    const int64_t all_rows = p->rows_cap;
    const int64_t nt = p->nt_cap > 0 ? p->nt_cap : 1;

    // One allocation, every array 256-byte aligned.
    struct Part {
        void **dst;
        size_t bytes;
    } parts[] = {
        {reinterpret_cast<void **>(&p->cnt), sizeof(int32_t) * E},
        {reinterpret_cast<void **>(&p->expert_off), sizeof(int32_t) * (E + 1)},
        {reinterpret_cast<void **>(&p->rcnt), sizeof(int32_t) * R},
        {reinterpret_cast<void **>(&p->rank_off), sizeof(int32_t) * (R + 1)},
        {reinterpret_cast<void **>(&p->rtok_off), sizeof(int32_t) * (R + 1)},
        {reinterpret_cast<void **>(&p->slot), sizeof(int32_t) * (rows > 0 ? rows : 1)},
        {reinterpret_cast<void **>(&p->src_tok), sizeof(int32_t) * (all_rows > 0 ? all_rows : 1)},
        {reinterpret_cast<void **>(&p->src_j), sizeof(int32_t) * (all_rows > 0 ? all_rows : 1)},
        {reinterpret_cast<void **>(&p->rtok), sizeof(int32_t) * (p->rtok_cap > 0 ? p->rtok_cap : 1)},
        {reinterpret_cast<void **>(&p->fanout), sizeof(uint32_t) * (p->rtok_cap > 0 ? p->rtok_cap : 1)},
        {reinterpret_cast<void **>(&p->err), sizeof(uint32_t)},
        {reinterpret_cast<void **>(&p->sync), 2 * sizeof(uint32_t)},
        {reinterpret_cast<void **>(&p->tile_cnt), sizeof(int32_t) * E * nt},
        {reinterpret_cast<void **>(&p->tile_rcnt), sizeof(int32_t) * R * nt},
        {reinterpret_cast<void **>(&p->tile_err), sizeof(uint32_t) * nt},
        {reinterpret_cast<void **>(&p->group_flag), sizeof(uint32_t) * (nt + 16)},
        {reinterpret_cast<void **>(&p->work), 4 * sizeof(uint32_t)},
        {reinterpret_cast<void **>(&p->ready), sizeof(uint32_t) * (max_tokens > 0 ? max_tokens : 1)},
    };
    size_t total = 0;
    for (const Part &part : parts)
        total += align256(part.bytes);
    void *mem = nullptr;
    cudaError_t e = cudaMalloc(&mem, total);
    if (e != cudaSuccess) {
        delete p;
        (void)cudaGetLastError();
        return fail(e == cudaErrorMemoryAllocation ? MOE_ENOMEM : MOE_ECUDA,
                    "cudaMalloc(%zu): %s", total, cudaGetErrorString(e));
    }
    e = cudaMemset(mem, 0, total);
    if (e != cudaSuccess) {
        cudaFree(mem);
        delete p;
        return cuda_fail(e, "cudaMemset");
    }
    size_t off = 0;
    for (const Part &part : parts) {
        *part.dst = static_cast<char *>(mem) + off;
        off += align256(part.bytes);
    }
    p->mem = mem;
    p->mem_bytes = total;
    *out = p;
    return ok();
}

moe_status moe_plan(const int32_t *topk_idx, const float *topk_w, int32_t N, int32_t k, int32_t E,
                    int32_t R, void *stream, moe_plan_t *plan)
{
    if (!plan)
        return fail(MOE_EINVAL, "plan must not be NULL");
    moe_status st = check_shape(N, k, E, R);
    if (st != MOE_OK)
        return st;
    if (N > 0 && (!topk_idx || !topk_w))
        return fail(MOE_EINVAL, "topk_idx and topk_w must not be NULL when N > 0");
    if (!aligned(topk_idx, 4) || !aligned(topk_w, 4))
        return fail(MOE_EINVAL, "topk_idx and topk_w must be 4-byte aligned");
    if (*plan) {
        moe_plan_s *p = *plan;
        if (p->k != k || p->E != E || p->R != R)
            return fail(MOE_EINVAL,
                        "plan was created for (k=%d, E=%d, R=%d), called with (k=%d, E=%d, R=%d)",
                        p->k, p->E, p->R, k, E, R);
        if (N > p->cap)
            return fail(MOE_EINVAL,
                        "plan capacity is %d tokens, called with N=%d (create a larger plan "
                        "with moe_plan_create)",
                        p->cap, N);
        if ((st = check_plan_device(p)) != MOE_OK)
            return st;
    } else {
        if ((st = moe_plan_create(N, k, E, R, plan)) != MOE_OK)
            return st;
    }
    moe_plan_s *p = *plan;
    p->N = N;
    p->topk_w = topk_w;
    cudaError_t e = moe::launch_plan(p, topk_idx, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess)
        return cuda_fail(e, "plan kernels");
    return ok();
}

// Checks a dispatch call and fills its kernel arguments.
static moe_status dispatch_args(const void *x, moe_dtype dtype, const float *x_scale, int32_t H,
                                moe_plan_t plan, void *recv, float *recv_scale,
                                moe::DispatchArgs *a)
{
    if (!plan)
        return fail(MOE_EINVAL, "plan must not be NULL");
    moe_plan_s *p = plan;
    if (H <= 0 || H > (1 << 24))
        return fail(MOE_EINVAL, "H must be in [1, 2^24] (got %d)", H);
    uint32_t elem = 0, srow = 0;
    if (dtype == MOE_BF16) {
        if (H % 8 != 0)
            return fail(MOE_EINVAL, "bf16 rows need H %% 8 == 0 (got H=%d)", H);
        if (x_scale || recv_scale)
            return fail(MOE_EINVAL, "bf16 dispatch takes no scales");
        elem = 2;
    } else if (dtype == MOE_FP8E4M3) {
        if (H % 128 != 0)
            return fail(MOE_EINVAL, "fp8 rows need H %% 128 == 0 (got H=%d)", H);
        if (p->N > 0 && (!x_scale || !recv_scale))
            return fail(MOE_EINVAL, "fp8 dispatch needs x_scale and recv_scale");
        elem = 1;
        srow = static_cast<uint32_t>(4 * (H / 128));
        const size_t sa = (srow % 16 == 0) ? 16 : 4;
        if (!aligned(x_scale, sa) || !aligned(recv_scale, sa))
            return fail(MOE_EINVAL, "scale arrays must be %zu-byte aligned", sa);
    } else {
        return fail(MOE_EINVAL, "unknown dtype %d", static_cast<int>(dtype));
    }
    if (p->N > 0 && (!x || !recv))
        return fail(MOE_EINVAL, "x and recv must not be NULL");
    if (!aligned(x, 16) || !aligned(recv, 16))
        return fail(MOE_EINVAL, "x and recv must be 16-byte aligned");
    moe_status st = check_plan_device(p);
    if (st != MOE_OK)
        return st;
    a->x = static_cast<const uint8_t *>(x);
    a->xs = reinterpret_cast<const uint8_t *>(x_scale);
    a->recv = static_cast<uint8_t *>(recv);
    a->rs = reinterpret_cast<uint8_t *>(recv_scale);
    a->slot = p->slot;
    a->err = p->err;
    a->N = p->N;
    a->k = p->k;
    a->n_rows = static_cast<int32_t>(moe::recv_rows(p->N, p->k, p->E, p->align));
    a->row_bytes = static_cast<uint32_t>(H) * elem;
    a->srow_bytes = srow;
    return MOE_OK;
}

moe_status moe_dispatch(const void *x, moe_dtype dtype, const float *x_scale, int32_t H,
                        moe_plan_t plan, void *recv, float *recv_scale, void *stream)
{
    moe::DispatchArgs a;
    moe_status st = dispatch_args(x, dtype, x_scale, H, plan, recv, recv_scale, &a);
    if (st != MOE_OK)
        return st;
    cudaError_t e = moe::launch_dispatch(a, plan->device, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess)
        return cuda_fail(e, "dispatch kernel");
    return ok();
}

// Checks a combine call and fills its kernel arguments.
static moe_status combine_args(const void *y, int32_t H, moe_plan_t plan, void *out, bool ranked,
                               moe::CombineArgs *a)
{
    if (!plan)
        return fail(MOE_EINVAL, "plan must not be NULL");
    moe_plan_s *p = plan;
    if (H <= 0 || H > (1 << 24) || H % 8 != 0)
        return fail(MOE_EINVAL, "H must be a multiple of 8 in [8, 2^24] (got %d)", H);
    if (p->N > 0 && (!y || !out || !p->topk_w))
        return fail(MOE_EINVAL, "y, out and the plan's weights must not be NULL");
    if (!aligned(y, 16) || !aligned(out, 16))
        return fail(MOE_EINVAL, "y and out must be 16-byte aligned");
    moe_status st = check_plan_device(p);
    if (st != MOE_OK)
        return st;
    a->y = static_cast<const uint16_t *>(y);
    a->slot = p->slot;
    a->w = p->topk_w;
    a->out = static_cast<uint16_t *>(out);
    a->err = p->err;
    a->N = p->N;
    a->k = p->k;
    a->n_rows = static_cast<int32_t>(moe::recv_rows(p->N, p->k, p->E, p->align));
    a->H = H;
    a->rank_off = p->rank_off;
    a->R = p->R;
    a->ranked = ranked;
    return MOE_OK;
}

static moe_status combine_impl(const void *y, int32_t H, moe_plan_t plan, void *out, void *stream,
                               bool ranked)
{
    moe::CombineArgs a;
    moe_status st = combine_args(y, H, plan, out, ranked, &a);
    if (st != MOE_OK)
        return st;
    cudaError_t e = moe::launch_combine(a, plan->device, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess)
        return cuda_fail(e, "combine kernel");
    return ok();
}

moe_status moe_dispatch_combine(const void *x, moe_dtype dtype, const float *x_scale,
                                int32_t H_x, moe_plan_t dispatch_plan, void *recv,
                                float *recv_scale, const void *y, int32_t H_y,
                                moe_plan_t combine_plan, void *out, int32_t ranked, void *stream)
{
    moe::FusedArgs f;
    moe_status st =
        dispatch_args(x, dtype, x_scale, H_x, dispatch_plan, recv, recv_scale, &f.d);
    if (st != MOE_OK)
        return st;
    st = combine_args(y, H_y, combine_plan, out, ranked != 0, &f.c);
    if (st != MOE_OK)
        return st;
    if (dispatch_plan->device != combine_plan->device)
        return fail(MOE_EINVAL, "both plans must be on the same device");
    if (f.d.srow_bytes % 16 != 0)
        return fail(MOE_EINVAL,
                    "fused dispatch needs fp8 scale rows of a multiple of 16 bytes "
                    "(H %% 512 == 0; got H=%d)",
                    H_x);
    // The combine may read the rows this call dispatches only as a whole: the same buffer
    // laid out by the same plan, in which case each token waits for its own dispatch.
    const uintptr_t r0 = reinterpret_cast<uintptr_t>(recv);
    const uintptr_t r1 = r0 + static_cast<uintptr_t>(f.d.n_rows) * f.d.row_bytes;
    const uintptr_t y0 = reinterpret_cast<uintptr_t>(y);
    const uintptr_t y1 = y0 + static_cast<uintptr_t>(f.c.n_rows) * static_cast<uintptr_t>(f.c.H) * 2u;
    const bool depends = y0 == r0 && f.d.N > 0 && f.c.N > 0;
    if (depends && (combine_plan != dispatch_plan || dtype != MOE_BF16 || H_x != H_y))
        return fail(MOE_EINVAL, "y == recv needs one plan, bf16 rows and H_x == H_y");
    if (!depends && f.d.N > 0 && f.c.N > 0 && y0 < r1 && r0 < y1)
        return fail(MOE_EINVAL, "y and recv overlap without being the same buffer");
    // Small calls: the two kernels back to back (stream order also covers y == recv).
    // Measured on B200: the one-launch kernel starts to win between 250 and 500 MB.
    const double traffic_kb =
        (static_cast<double>(f.d.N) * (f.d.row_bytes + f.d.srow_bytes) * (1 + f.d.k) +
         static_cast<double>(f.c.N) * f.c.H * 2.0 * (1 + f.c.k)) / 1024.0;
    const int min_kb = moe::tuning().fused_min_kb > 0 ? moe::tuning().fused_min_kb : 320 * 1024;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (traffic_kb < min_kb) {
        cudaError_t e = moe::launch_dispatch(f.d, dispatch_plan->device, s);
        if (e != cudaSuccess)
            return cuda_fail(e, "dispatch kernel");
        e = moe::launch_combine(f.c, combine_plan->device, s);
        if (e != cudaSuccess)
            return cuda_fail(e, "combine kernel");
        return ok();
    }
    f.work = dispatch_plan->work;
    f.ready = dispatch_plan->ready;
    f.ready_len = static_cast<uint32_t>(dispatch_plan->cap);
    f.use_flags = depends;
    cudaError_t e = moe::launch_fused(f, dispatch_plan->device, s);
    if (e != cudaSuccess)
        return cuda_fail(e, "fused dispatch/combine kernel");
    return ok();
}

moe_status moe_combine(const void *y, int32_t H, moe_plan_t plan, void *out, void *stream)
{
    return combine_impl(y, H, plan, out, stream, false);
}

moe_status moe_combine_ranked(const void *y, int32_t H, moe_plan_t plan, void *out, void *stream)
{
    return combine_impl(y, H, plan, out, stream, true);
}

moe_status moe_plan_query(moe_plan_t plan, moe_plan_view *v)
{
    if (!plan || !v)
        return fail(MOE_EINVAL, "plan and view must not be NULL");
    const moe_plan_s *p = plan;
    v->N = p->N;
    v->k = p->k;
    v->E = p->E;
    v->R = p->R;
    v->experts_per_rank = p->epr;
    v->capacity_tokens = p->cap;
    v->cnt = p->cnt;
    v->expert_off = p->expert_off;
    v->rcnt = p->rcnt;
    v->rank_off = p->rank_off;
    v->rtok_off = p->rtok_off;
    v->slot = p->slot;
    v->src_tok = p->src_tok;
    v->src_j = p->src_j;
    v->rtok = p->rtok;
    v->fanout = p->fanout;
    v->err = p->err;
    v->topk_w = p->topk_w;
    v->plan_kernels = p->plan_kernels;
    v->plan_kind = p->plan_kind;
    v->dedup_lists = p->dedup_lists ? 1 : 0;
    v->align = p->align;
    v->recv_rows = static_cast<int32_t>(moe::recv_rows(p->N, p->k, p->E, p->align));
    return ok();
}

moe_status moe_plan_check(moe_plan_t plan, void *stream, uint32_t *flags)
{
    if (!plan || !flags)
        return fail(MOE_EINVAL, "plan and flags must not be NULL");
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess)
        return cuda_fail(e, "cudaStreamSynchronize");
    e = cudaMemcpy(flags, plan->err, sizeof(uint32_t), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess)
        return cuda_fail(e, "cudaMemcpy(err)");
    if (*flags & MOE_ERR_TIMEOUT) {
        // a grid barrier was abandoned: rearm its words (and clear the error word, which
        // keeps a timeout until it has been reported here) for the next plan
        e = cudaMemset(plan->sync, 0, 2 * sizeof(uint32_t));
        if (e == cudaSuccess)
            e = cudaMemset(plan->err, 0, sizeof(uint32_t));
        if (e == cudaSuccess)
            e = cudaMemset(plan->group_flag, 0,
                           sizeof(uint32_t) * ((plan->nt_cap > 0 ? plan->nt_cap : 1) + 16));
        if (e != cudaSuccess)
            return cuda_fail(e, "cudaMemset(sync)");
        // and the fused kernel's work words, with its flags (the epoch starts again)
        e = cudaMemset(plan->work, 0, 4 * sizeof(uint32_t));
        if (e == cudaSuccess)
            e = cudaMemset(plan->ready, 0, sizeof(uint32_t) * (plan->cap > 0 ? plan->cap : 1));
        if (e != cudaSuccess)
            return cuda_fail(e, "cudaMemset(work, ready)");
    }
    return ok();
}

moe_status moe_wait_selftest(int32_t which, void *stream, uint32_t *flags)
{
    if (!flags)
        return fail(MOE_EINVAL, "flags must not be NULL");
    if (which < 0 || which > 3)
        return fail(MOE_EINVAL,
                    "which must be 0 (flag wait), 1 (mbarrier wait), 2 (grid barrier) or 3 "
                    "(group exchange), got %d",
                    which);
    cudaError_t e = moe::run_wait_selftest(which, static_cast<cudaStream_t>(stream), flags);
    if (e != cudaSuccess)
        return cuda_fail(e, "wait self-test");
    return ok();
}

moe_status moe_plan_destroy(moe_plan_t plan)
{
    if (!plan)
        return ok();
    cudaError_t e = cudaSuccess;
    if (plan->mem)
        e = cudaFree(plan->mem);
    delete plan;
    if (e != cudaSuccess)
        return cuda_fail(e, "cudaFree");
    return ok();
}

}  // extern "C"
