/*
 * CPU oracle for the MoE token shuffle -- TEST INFRASTRUCTURE ONLY.
 *
 * Only the tests, the package smoke check and the benchmark's CPU-baseline leg may
 * load this library.  The CUDA library never links, includes or calls it, and this
 * file includes nothing from the CUDA library.
 *
 * Each function is the plain definition of one step, written as slow scalar loops with
 * no blocking, fusion or reordering:
 *
 *   plan      -- FUSCO (arXiv 2512.22036), abstract: the layout is captured as
 *                fine-grained logical segments and placement follows from it; the
 *                FUSCO summary (reportify "FUSCO" page), Group 3: the interface is built
 *                around logical segments so data is placed directly, with no staging or
 *                post-rearrangement.  Segments are per-expert runs of the receive
 *                buffer, grouped by rank; rows inside a segment keep ascending token
 *                order.  Dedup ("eliminating redundant communication", FUSCO abstract;
 *                the Token B example of the DySHARP blog, section 2): one move per
 *                (token, destination rank), listed per rank in ascending token order
 *                with a bitmask of the top-k columns it fans out to.
 *   dispatch  -- FUSCO abstract: the expert-major layout is produced while the data
 *                moves.  recv[slot[t,j]] = x[t] byte for byte (fp8 scales move with
 *                their row).
 *   combine   -- DySHARP blog, section 1 ("compute, then Combine back") and section 2
 *                (the partial results of one token are summed): out[t] =
 *                bf16_rne( fp32 fma chain over j = 0..k-1 of w[t,j] * y[slot[t,j]] ).
 *                The chain order and fp32 accumulation are fixed by the accuracy
 *                target; combine_f64 is the exact-order-free float64 sum used to bound
 *                the rounding error; combine_ranked reduces per rank first.
 *
 * Readings where the pages are silent: expert e lives on rank e / (E/R); segments are
 * tight unless an alignment is asked for, in which case each expert's segment starts on a
 * multiple of `align` rows and the rows after its entries are padding (no token); an id
 * of -1 marks an entry the router dropped (no receive row, no contribution, not an
 * error); other ids are distinct within a token and in [0, E) -- anything else is
 * rejected with ORACLE_EINVAL.  Build: gcc -O2 -ffp-contract=off (no contraction, so
 * every fma below is the only fused operation).
 *
 * The token loops of dispatch and combine carry an OpenMP pragma.  The oracle build
 * ignores it (no -fopenmp); a second build with -fopenmp (liboracle_omp.so) exists only
 * so the benchmark can also report the oracle's time on all host cores.  Each iteration
 * writes rows no other iteration writes (slots are distinct; out row t belongs to token
 * t), so both builds give identical bytes.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_EINVAL 1

static int valid_shape(int64_t N, int32_t k, int32_t E, int32_t R)
{
    if (N < 0 || k < 1 || k > 32 || E < 1 || R < 1 || k > E || E % R != 0)
        return 0;
    if (N * (int64_t)k >= ((int64_t)1 << 31))
        return 0;
    return 1;
}

#define DROPPED (-1)

/* 1 if every id is -1 (dropped) or in [0,E), and no token lists an expert twice. */
int oracle_validate(const int32_t *topk_idx, int64_t N, int32_t k, int32_t E)
{
    for (int64_t t = 0; t < N; ++t) {
        for (int32_t j = 0; j < k; ++j) {
            int32_t e = topk_idx[t * k + j];
            if (e == DROPPED)
                continue;
            if (e < 0 || e >= E)
                return 0;
            for (int32_t i = 0; i < j; ++i)
                if (topk_idx[t * k + i] == e)
                    return 0;
        }
    }
    return 1;
}

/* 1 when column j of token t is routed to an expert of rank r (dropped entries are not). */
static int on_rank(const int32_t *topk_idx, int64_t t, int32_t j, int32_t k, int32_t epr,
                   int32_t r)
{
    int32_t e = topk_idx[t * k + j];
    return e != DROPPED && e / epr == r;
}

/* Number of (token, rank) moves: tokens counted once per distinct rank they touch. */
int64_t oracle_dedup_count(const int32_t *topk_idx, int64_t N, int32_t k, int32_t E, int32_t R)
{
    int32_t epr = E / R;
    int64_t total = 0;
    for (int32_t r = 0; r < R; ++r)
        for (int64_t t = 0; t < N; ++t) {
            int hit = 0;
            for (int32_t j = 0; j < k; ++j)
                if (on_rank(topk_idx, t, j, k, epr, r))
                    hit = 1;
            total += hit;
        }
    return total;
}

/*
 * Outputs (all caller-allocated):
 *   cnt[E]          entries routed to each expert (dropped entries excluded)
 *   expert_off[E+1] segment starts, expert-major: expert_off[e+1] = expert_off[e] +
 *                   cnt[e] rounded up to a multiple of `align`
 *   rcnt[R]         tokens with at least one expert on rank r (dedup moves)
 *   rank_off[R+1]   first receive row of each rank = expert_off[r * E/R]
 *   rtok_off[R+1]   exclusive prefix sum of rcnt
 *   slot[N*k]       receive row of entry (t,j): expert_off[e] + #{t' < t routed to e},
 *                   or -1 for a dropped entry
 *   src_tok[rows]   token of each receive row, -1 for padding and unused rows
 *   src_j[rows]     top-k column of each receive row, -1 for padding and unused rows
 *   rtok[cap]       rtok[rtok_off[r] + i] = i-th smallest token touching rank r
 *   fanout[cap]     bit j set when column j of that token is an expert of rank r
 * rows = N*k + E*(align - 1), the receive rows a buffer must hold.
 */
int oracle_plan_ex(const int32_t *topk_idx, int64_t N, int32_t k, int32_t E, int32_t R,
                   int32_t align, int32_t *cnt, int32_t *expert_off, int32_t *rcnt,
                   int32_t *rank_off, int32_t *rtok_off, int32_t *slot, int32_t *src_tok,
                   int32_t *src_j, int32_t *rtok, uint32_t *fanout, int64_t rtok_cap)
{
    if (!valid_shape(N, k, E, R) || align < 1 || !oracle_validate(topk_idx, N, k, E))
        return ORACLE_EINVAL;
    const int32_t epr = E / R;
    const int64_t rows = N * k + (int64_t)E * (align - 1);

    /* histogram over experts */
    for (int32_t e = 0; e < E; ++e)
        cnt[e] = 0;
    for (int64_t t = 0; t < N; ++t)
        for (int32_t j = 0; j < k; ++j)
            if (topk_idx[t * k + j] != DROPPED)
                cnt[topk_idx[t * k + j]] += 1;

    /* exclusive scan of the (aligned) segment sizes: segment starts */
    expert_off[0] = 0;
    for (int32_t e = 0; e < E; ++e)
        expert_off[e + 1] = expert_off[e] + (cnt[e] + align - 1) / align * align;
    for (int32_t r = 0; r <= R; ++r)
        rank_off[r] = expert_off[r * epr];

    /* stable rank inside each segment: tokens in ascending order */
    for (int64_t i = 0; i < rows; ++i) {
        src_tok[i] = -1;
        src_j[i] = -1;
    }
    int32_t *fill = (int32_t *)calloc((size_t)E, sizeof(int32_t));
    if (!fill)
        return ORACLE_EINVAL;
    for (int64_t t = 0; t < N; ++t)
        for (int32_t j = 0; j < k; ++j) {
            int32_t e = topk_idx[t * k + j];
            if (e == DROPPED) {
                slot[t * k + j] = -1;
                continue;
            }
            int32_t s = expert_off[e] + fill[e];
            fill[e] += 1;
            slot[t * k + j] = s;
            src_tok[s] = (int32_t)t;
            src_j[s] = j;
        }
    free(fill);

    /* dedup: one move per (token, rank), tokens ascending inside each rank */
    rtok_off[0] = 0;
    for (int32_t r = 0; r < R; ++r) {
        int32_t n = 0;
        for (int64_t t = 0; t < N; ++t) {
            uint32_t mask = 0;
            for (int32_t j = 0; j < k; ++j)
                if (on_rank(topk_idx, t, j, k, epr, r))
                    mask |= 1u << j;
            if (mask) {
                int64_t pos = (int64_t)rtok_off[r] + n;
                if (pos >= rtok_cap)
                    return ORACLE_EINVAL;
                rtok[pos] = (int32_t)t;
                fanout[pos] = mask;
                n += 1;
            }
        }
        rcnt[r] = n;
        rtok_off[r + 1] = rtok_off[r] + n;
    }
    return ORACLE_OK;
}

/* The plan with tight segments (align = 1). */
int oracle_plan(const int32_t *topk_idx, int64_t N, int32_t k, int32_t E, int32_t R,
                int32_t *cnt, int32_t *expert_off, int32_t *rcnt, int32_t *rank_off,
                int32_t *rtok_off, int32_t *slot, int32_t *src_tok, int32_t *src_j,
                int32_t *rtok, uint32_t *fanout, int64_t rtok_cap)
{
    return oracle_plan_ex(topk_idx, N, k, E, R, 1, cnt, expert_off, rcnt, rank_off, rtok_off,
                          slot, src_tok, src_j, rtok, fanout, rtok_cap);
}

/*
 * recv[slot[t,j]] = x[t] for every entry; row_bytes payload bytes per row.  With
 * scale_bytes > 0 the per-row scale block x_scale[t] moves to recv_scale[slot[t,j]].
 */
void oracle_dispatch(const uint8_t *x, const uint8_t *x_scale, const int32_t *slot,
                     int64_t N, int32_t k, int64_t row_bytes, int64_t scale_bytes,
                     uint8_t *recv, uint8_t *recv_scale)
{
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < N; ++t)
        for (int32_t j = 0; j < k; ++j) {
            int64_t s = slot[t * k + j];
            if (s < 0)
                continue; /* dropped entry: no receive row */
            memcpy(recv + s * row_bytes, x + t * row_bytes, (size_t)row_bytes);
            if (scale_bytes > 0)
                memcpy(recv_scale + s * scale_bytes, x_scale + t * scale_bytes,
                       (size_t)scale_bytes);
        }
}

static float bf16_to_f32(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* IEEE round-to-nearest-even of a float32 to its top 16 bits (bfloat16). */
static uint16_t f32_to_bf16_rne(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu))
        return (uint16_t)((u >> 16) | 0x0040u); /* quiet NaN, sign kept */
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

/* out[t,c] = bf16_rne(acc), acc = fma(w[t,j], y[slot[t,j],c], acc) for j = 0..k-1, acc0 = +0 */
void oracle_combine(const uint16_t *y, const int32_t *slot, const float *w, int64_t N,
                    int32_t k, int64_t H, uint16_t *out)
{
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < N; ++t)
        for (int64_t c = 0; c < H; ++c) {
            float acc = 0.0f;
            for (int32_t j = 0; j < k; ++j) {
                int64_t s = slot[t * k + j];
                if (s < 0)
                    continue; /* dropped entry contributes nothing */
                acc = fmaf(w[t * k + j], bf16_to_f32(y[s * H + c]), acc);
            }
            out[t * H + c] = f32_to_bf16_rne(acc);
        }
}

/*
 * Rank-grouped combine (the combine-side counterpart of the per-rank dedup; DySHARP blog,
 * section 2: the partial results that several destinations produce for one token could be
 * summed before they travel back, and section 5: dymultimem.ld_reduce returns one reduced
 * result).  For each rank r in ascending order that holds some expert of token t, the
 * rank's partial is the fp32 fma chain over the token's columns on r in ascending column
 * order, starting from +0; the partials are then added in ascending rank order in fp32,
 * starting from +0; the result is rounded to bf16 (nearest even).
 */
void oracle_combine_ranked(const uint16_t *y, const int32_t *slot, const float *w,
                           const int32_t *topk_idx, int64_t N, int32_t k, int64_t H, int32_t E,
                           int32_t R, uint16_t *out)
{
    const int32_t epr = E / R;
    for (int64_t t = 0; t < N; ++t)
        for (int64_t c = 0; c < H; ++c) {
            float total = 0.0f;
            for (int32_t r = 0; r < R; ++r) {
                int any = 0;
                float part = 0.0f;
                for (int32_t j = 0; j < k; ++j) {
                    if (!on_rank(topk_idx, t, j, k, epr, r))
                        continue;
                    int64_t s = slot[t * k + j];
                    part = fmaf(w[t * k + j], bf16_to_f32(y[s * H + c]), part);
                    any = 1;
                }
                if (any)
                    total = total + part;
            }
            out[t * H + c] = f32_to_bf16_rne(total);
        }
}

/* Float64 sum of w[t,j] * y[slot[t,j],c] (no bf16 rounding): the reference value for
 * rounding-error bounds.  Each product of a float32 weight and a bf16 value is exact in
 * float64 (24 + 8 significant bits). */
void oracle_combine_f64(const uint16_t *y, const int32_t *slot, const float *w, int64_t N,
                        int32_t k, int64_t H, double *out)
{
    for (int64_t t = 0; t < N; ++t)
        for (int64_t c = 0; c < H; ++c) {
            double acc = 0.0;
            for (int32_t j = 0; j < k; ++j) {
                int64_t s = slot[t * k + j];
                if (s < 0)
                    continue;
                acc += (double)w[t * k + j] * (double)bf16_to_f32(y[s * H + c]);
            }
            out[t * H + c] = acc;
        }
}

/* bf16 round-to-nearest-even of float32 values (exposed so tests can pin the rounding). */
void oracle_f32_to_bf16(const float *in, int64_t n, uint16_t *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = f32_to_bf16_rne(in[i]);
}
