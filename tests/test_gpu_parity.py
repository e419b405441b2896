"""Parity of the CUDA path with the CPU oracle on the same seeded inputs.

Plan and dispatch must match bit for bit; combine must be within 1 bf16 ulp, max abs 1e-2
and max rel 8e-3 (and, since both sides run the same fp32 fma chain, is expected to
match bit for bit as well).  Full-size cases run in the launch configuration the
benchmark times (the library defaults)."""

import numpy as np
import pytest
import torch

import oracle
from tests.shuffle_cases import (
    assert_combine_close, assert_plan_equal, bits16, bits_to_f32, gpu_plan, make_inputs,
    plan_to_host,
)
from tests.test_oracle_plan import drop_some
from workloads import CONFIGS, make_routing

pytestmark = pytest.mark.gpu

ALL = ["tiny", "mixtral", "dsv3", "skew", "long"]


def run_all(cfg, seed, y_identity=False):
    """GPU plan/dispatch/combine and oracle plan/dispatch/combine; returns both sides."""
    import moe_expert_shuffling_b200 as ms
    idx, w, x, xs, y = make_inputs(cfg, seed, y=not y_identity)
    p, ti, tw = gpu_plan(idx, w, cfg.E, cfg.R)
    if cfg.payload == "fp8":
        recv, rs = ms.moe_dispatch(x, p, x_scale=xs)
    else:
        recv, rs = ms.moe_dispatch(x, p), None
    yy = recv if y_identity else y
    out = ms.moe_combine(yy, p)
    torch.cuda.synchronize()
    assert p.check() == 0

    ref = oracle.plan(idx, cfg.E, cfg.R)
    gp = plan_to_host(p)
    x_h = x.cpu()
    if cfg.payload == "fp8":
        ref_recv, ref_rs = oracle.dispatch(x_h.numpy(), ref.slot, xs.cpu().numpy())
        got_recv = recv.cpu().numpy()
        got_rs = rs.cpu().numpy().view(np.uint8)
    else:
        ref_recv = oracle.dispatch(bits16(x_h).view(np.uint8).reshape(cfg.N, -1), ref.slot)
        ref_rs = got_rs = None
        got_recv = bits16(recv).view(np.uint8).reshape(cfg.N * cfg.k, -1)
    y_h = ref_recv.view(np.uint16).reshape(cfg.N * cfg.k, cfg.H) if y_identity else bits16(y)
    ref_out = oracle.combine(y_h, ref.slot, w)
    return dict(gp=gp, ref=ref, got_recv=got_recv, ref_recv=ref_recv, got_rs=got_rs,
                ref_rs=ref_rs, got_out=bits16(out), ref_out=ref_out, x=x_h)


@pytest.mark.parametrize("name", ALL)
def test_full_size_parity(name):
    cfg = CONFIGS[name]
    r = run_all(cfg, 0, y_identity=(cfg.y == "identity"))
    assert_plan_equal(r["gp"], r["ref"])
    assert np.array_equal(r["got_recv"], r["ref_recv"])
    if r["ref_rs"] is not None:
        assert np.array_equal(r["got_rs"], r["ref_rs"])
    assert_combine_close(r["got_out"], r["ref_out"])
    assert np.array_equal(r["got_out"], r["ref_out"])


@pytest.mark.parametrize("name,seed", [("tiny", 1), ("tiny", 2), ("dsv3", 1), ("skew", 2)])
def test_more_seeds(name, seed):
    cfg = CONFIGS[name]
    if name in ("dsv3", "skew"):
        cfg = cfg.with_tokens(3000)   # several tiles plus a ragged tail
    r = run_all(cfg, seed)
    assert_plan_equal(r["gp"], r["ref"])
    assert np.array_equal(r["got_recv"], r["ref_recv"])
    assert np.array_equal(r["got_out"], r["ref_out"])


@pytest.mark.parametrize("name", ["dsv3_k16", "dsv3_k32"])
def test_wide_topk_parity(name):
    """Top-16 and top-32 of 256 experts (the wider-fan-out settings), 4096 tokens."""
    cfg = CONFIGS[name].with_tokens(4096)
    r = run_all(cfg, 0)
    assert_plan_equal(r["gp"], r["ref"])
    assert np.array_equal(r["got_recv"], r["ref_recv"])
    assert_combine_close(r["got_out"], r["ref_out"])
    assert np.array_equal(r["got_out"], r["ref_out"])


@pytest.mark.parametrize("cfg", [
    CONFIGS["dsv3"].with_tokens(2000),
    CONFIGS["skew"].with_tokens(1000),
    CONFIGS["long"].with_tokens(3000),
    CONFIGS["mixtral"].with_tokens(1000),
    CONFIGS["tiny"],
    CONFIGS["dsv3_k16"].with_tokens(500),
    CONFIGS["dsv3_k32"].with_tokens(500),
    CONFIGS["dsv3"].replace(N=300, H=64, E=1024, k=8, R=1024),
    CONFIGS["dsv3"].replace(N=300, H=64, E=1024, k=8, R=1),
], ids=lambda c: f"{c.name}-N{c.N}-E{c.E}-k{c.k}-R{c.R}")
def test_ranked_combine_parity(cfg):
    """moe_combine_ranked matches the oracle's rank-grouped order bit for bit."""
    import moe_expert_shuffling_b200 as ms
    idx, w, x, xs, y = make_inputs(cfg, 3)
    p, ti, tw = gpu_plan(idx, w, cfg.E, cfg.R)
    out = ms.moe_combine(y, p, ranked=True)
    torch.cuda.synchronize()
    ref = oracle.plan(idx, cfg.E, cfg.R)
    want = oracle.combine_ranked(bits16(y), ref.slot, w, idx, cfg.E, cfg.R)
    got = bits16(out)
    assert_combine_close(got, want)
    assert np.array_equal(got, want)


@pytest.mark.parametrize("name", ["mixtral", "dsv3"])
def test_identity_experts_return_x(name):
    """combine(dispatch(x)) == x with y = recv and weights summing to 1."""
    cfg = CONFIGS[name]
    r = run_all(cfg, 0, y_identity=True)
    assert np.array_equal(bits_to_f32(r["got_out"]), bits_to_f32(bits16(r["x"])))


@pytest.mark.parametrize("cfg", [
    CONFIGS["tiny"].with_tokens(1),
    CONFIGS["tiny"].with_tokens(127),
    CONFIGS["tiny"].with_tokens(129),
    CONFIGS["dsv3"].with_tokens(1000).replace(H=256),
    CONFIGS["tiny"].replace(k=1, N=777),                                   # top-1
    CONFIGS["dsv3"].replace(N=300, H=64, E=64, k=32, R=8),                 # maximum k
    CONFIGS["dsv3"].replace(N=400, H=64, E=1024, k=8, R=1024),             # maximum E, E == R
    CONFIGS["dsv3"].replace(N=400, H=64, E=1024, k=8, R=1),                # one rank
    CONFIGS["tiny"].replace(N=200, H=8),                                   # smallest bf16 row
    CONFIGS["tiny"].replace(N=70, H=20000),                                # row split in chunks
    CONFIGS["long"].replace(N=300, H=128),                                 # 4-byte scale rows
    CONFIGS["long"].replace(N=300, H=640),                                 # 20-byte scale rows
    CONFIGS["long"].replace(N=50, H=65536),                                # chunked fp8 row
    CONFIGS["long"].replace(N=1000, H=512, k=4, E=16, R=16),
], ids=lambda c: f"{c.name}-N{c.N}-H{c.H}-E{c.E}-k{c.k}-R{c.R}-{c.payload}")
def test_edge_shapes(cfg):
    r = run_all(cfg, 0)
    assert_plan_equal(r["gp"], r["ref"])
    assert np.array_equal(r["got_recv"], r["ref_recv"])
    if r["ref_rs"] is not None:
        assert np.array_equal(r["got_rs"], r["ref_rs"])
    assert_combine_close(r["got_out"], r["ref_out"])
    assert np.array_equal(r["got_out"], r["ref_out"])


def test_empty_input():
    import moe_expert_shuffling_b200 as ms
    ti = torch.zeros((0, 8), dtype=torch.int32, device="cuda")
    tw = torch.zeros((0, 8), dtype=torch.float32, device="cuda")
    p = ms.moe_plan(ti, tw, 256, 32)
    recv = ms.moe_dispatch(torch.zeros((0, 64), dtype=torch.bfloat16, device="cuda"), p)
    out = ms.moe_combine(recv, p)
    assert recv.shape == (0, 64) and out.shape == (0, 64)
    assert p.check() == 0
    a = p.arrays()
    assert int(a["expert_off"].abs().sum()) == 0 and int(a["rtok_off"].abs().sum()) == 0


def test_plan_reuse_and_capacity():
    import moe_expert_shuffling_b200 as ms
    cfg = CONFIGS["dsv3"].with_tokens(2000)
    p = ms.moe_plan_create(2000, cfg.k, cfg.E, cfg.R)
    for seed, N in ((0, 2000), (1, 1500), (2, 129)):
        c = cfg.with_tokens(N)
        idx, w, x, _, y = make_inputs(c, seed)
        p, ti, tw = gpu_plan(idx, w, c.E, c.R, plan=p)
        recv = ms.moe_dispatch(x, p)
        out = ms.moe_combine(y, p)
        ref = oracle.plan(idx, c.E, c.R)
        assert_plan_equal(plan_to_host(p), ref)
        ref_recv = oracle.dispatch(bits16(x).view(np.uint8).reshape(N, -1), ref.slot)
        assert np.array_equal(bits16(recv).view(np.uint8).reshape(N * c.k, -1), ref_recv)
        assert np.array_equal(bits16(out), oracle.combine(bits16(y), ref.slot, w))
    idx, w, *_ = make_inputs(cfg.with_tokens(2001), 0, y=False)
    with pytest.raises(ms.MoeError, match="capacity"):
        gpu_plan(idx, w, cfg.E, cfg.R, plan=p)
    with pytest.raises(ms.MoeError, match="created for"):
        gpu_plan(idx[:10, :4].copy(), w[:10, :4].copy(), cfg.E, cfg.R, plan=p)


@pytest.mark.parametrize("cfg", [CONFIGS["tiny"].with_tokens(300),
                                 CONFIGS["dsv3_k32"].replace(N=300, H=64)],
                         ids=["tiny", "k32"])
@pytest.mark.parametrize("match", [1, 2], ids=["shuffles", "match"])
def test_invalid_routing_is_flagged_and_contained(cfg, match):
    """Out-of-range and repeated ids set error bits, get slot -1 and are skipped: plan,
    dispatch and combine equal, bit for bit, the oracle's on the routing with those entries
    marked dropped (-1).  Both ways of comparing a token's ids give the same."""
    import moe_expert_shuffling_b200 as ms
    idx, w, x, _, y = make_inputs(cfg, 0)
    bad = idx.copy()
    bad[3, 0] = cfg.E            # out of range
    bad[10, 1] = -5              # negative
    bad[20, 1] = bad[20, 0]      # repeated in one token (the first occurrence stays valid)
    bad[299, 0] = 2 ** 31 - 1
    ms.moe_tune("plan_match", match)
    try:
        p, ti, tw = gpu_plan(bad, w, cfg.E, cfg.R)
    finally:
        ms.moe_tune("plan_match", 0)
    recv = torch.zeros((cfg.N * cfg.k, cfg.H), dtype=torch.bfloat16, device="cuda")
    ms.moe_dispatch(x, p, recv=recv)
    out = ms.moe_combine(y, p)
    out_r = ms.moe_combine(y, p, ranked=True)
    flags = p.check()
    assert flags & ms.ERR_ID_RANGE and flags & ms.ERR_ID_DUP
    assert not flags & (ms.ERR_BOUNDS | ms.ERR_TIMEOUT)

    cleaned = bad.copy()
    for t, j in ((3, 0), (10, 1), (20, 1), (299, 0)):
        cleaned[t, j] = -1
    ref = oracle.plan(cleaned, cfg.E, cfg.R)
    g = plan_to_host(p)
    for name in ("cnt", "expert_off", "rcnt", "rank_off", "rtok_off", "slot", "src_tok",
                 "src_j", "rtok"):
        assert np.array_equal(g[name], getattr(ref, name)), name
    assert np.array_equal(g["fanout"], ref.fanout)
    assert int(g["cnt"].sum()) == int((cleaned >= 0).sum())
    used = ref.src_tok >= 0
    want_recv = oracle.dispatch(bits16(x).view(np.uint8).reshape(cfg.N, -1), ref.slot)
    got_recv = bits16(recv).view(np.uint8).reshape(cfg.N * cfg.k, -1)
    assert np.array_equal(got_recv[used], want_recv[used])
    assert not got_recv[~used].any()              # rows no entry maps to stay untouched
    yb = bits16(y)
    assert np.array_equal(bits16(out), oracle.combine(yb, ref.slot, w))
    assert np.array_equal(bits16(out_r), oracle.combine_ranked(yb, ref.slot, w, cleaned, cfg.E, cfg.R))


@pytest.mark.parametrize("knobs", [
    {"dispatch_stages": 2, "dispatch_lag": 1},
    {"dispatch_stages": 8, "dispatch_lag": 4, "dispatch_warps_per_cta": 2},
    {"dispatch_ctas_per_sm": 1, "combine_ctas_per_sm": 1},
    {"combine_stages": 2},
    {"plan_engine": 2},
    {"dispatch_units_per_warp": 10000, "combine_tokens_per_cta": 10000},
    {"combine_smem_kb": 64, "combine_ctas_per_sm": 2},
])
def test_launch_configuration_does_not_change_results(knobs):
    import moe_expert_shuffling_b200 as ms
    cfg = CONFIGS["dsv3"].with_tokens(1500)
    try:
        for k, v in knobs.items():
            ms.moe_tune(k, v)
        r = run_all(cfg, 2)
    finally:
        for k in knobs:
            ms.moe_tune(k, 0)
    assert_plan_equal(r["gp"], r["ref"])
    assert np.array_equal(r["got_recv"], r["ref_recv"])
    assert np.array_equal(r["got_out"], r["ref_out"])


def test_side_stream():
    import moe_expert_shuffling_b200 as ms
    cfg = CONFIGS["dsv3"].with_tokens(700)
    idx, w, x, _, y = make_inputs(cfg, 1)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        ti = torch.from_numpy(idx).cuda()
        tw = torch.from_numpy(w).cuda()
        p = ms.moe_plan(ti, tw, cfg.E, cfg.R)
        recv = ms.moe_dispatch(x, p)
        out = ms.moe_combine(y, p)
    s.synchronize()
    ref = oracle.plan(idx, cfg.E, cfg.R)
    assert np.array_equal(bits16(out), oracle.combine(bits16(y), ref.slot, w))


@pytest.mark.parametrize("name,N,frac,align", [
    ("tiny", 128, 0.2, 1), ("tiny", 300, 0.3, 8), ("dsv3", 2000, 0.1, 128),
    ("long", 3000, 0.05, 64), ("mixtral", 2000, 0.5, 16), ("dsv3", 700, 1.0, 4),
    ("dsv3_k32", 300, 0.2, 32),
])
def test_dropped_and_aligned_parity(name, N, frac, align):
    """Dropped entries (id -1) and aligned expert segments match the oracle bit for bit."""
    import moe_expert_shuffling_b200 as ms
    cfg = CONFIGS[name].with_tokens(N)
    idx, w, x, xs, _ = make_inputs(cfg, 5, y=False)
    idx = drop_some(idx, frac, 13)
    ref = oracle.plan(idx, cfg.E, cfg.R, align=align)
    p = ms.moe_plan_create(N, cfg.k, cfg.E, cfg.R, align=align)
    p, ti, tw = gpu_plan(idx, w, cfg.E, cfg.R, plan=p)
    assert p.rows == ref.rows and p.align == align
    got = plan_to_host(p)
    for name_ in ("cnt", "expert_off", "rcnt", "rank_off", "rtok_off", "slot", "src_tok",
                  "src_j", "rtok"):
        assert np.array_equal(got[name_], getattr(ref, name_)), name_
    assert np.array_equal(got["fanout"], ref.fanout)
    assert int(got["err"][0]) == 0                       # drops are not errors
    used = ref.src_tok >= 0
    if cfg.payload == "fp8":
        recv, rs = ms.moe_dispatch(x, p, x_scale=xs)
        ref_recv, ref_rs = oracle.dispatch(x.cpu().numpy(), ref.slot, xs.cpu().numpy(), rows=ref.rows)
        assert np.array_equal(rs.cpu().numpy().view(np.uint8)[used], ref_rs[used])
        got_recv = recv.cpu().numpy()
    else:
        recv = ms.moe_dispatch(x, p)
        ref_recv = oracle.dispatch(bits16(x).view(np.uint8).reshape(N, -1), ref.slot, rows=ref.rows)
        got_recv = bits16(recv).view(np.uint8).reshape(ref.rows, -1)
    assert np.array_equal(got_recv[used], ref_recv[used])
    g = torch.Generator(device="cuda")
    g.manual_seed(21)
    y = torch.randn((ref.rows, cfg.H), generator=g, device="cuda").to(torch.bfloat16)
    out = ms.moe_combine(y, p)
    out_r = ms.moe_combine(y, p, ranked=True)
    assert p.check() == 0
    yb = bits16(y)
    assert np.array_equal(bits16(out), oracle.combine(yb, ref.slot, w))
    assert np.array_equal(bits16(out_r), oracle.combine_ranked(yb, ref.slot, w, idx, cfg.E, cfg.R))


def test_drops_alone_raise_no_error():
    import moe_expert_shuffling_b200 as ms
    idx = -np.ones((257, 4), np.int32)
    w = np.full((257, 4), 0.25, np.float32)
    p, ti, tw = gpu_plan(idx, w, 16, 4)
    x = torch.randn((257, 64), device="cuda").to(torch.bfloat16)
    recv = ms.moe_dispatch(x, p)
    out = ms.moe_combine(recv, p)
    assert p.check() == 0
    assert not bits16(out).any()              # nothing routed: out is +0
    a = plan_to_host(p)
    assert np.all(a["slot"] == -1) and np.all(a["src_tok"] == -1) and a["cnt"].sum() == 0


@pytest.mark.parametrize("cfg,frac,align,kind", [
    (CONFIGS["dsv3"].with_tokens(128), 0.0, 1, "one_tile"),
    (CONFIGS["dsv3"].with_tokens(16), 0.25, 64, "one_tile"),
    (CONFIGS["dsv3"].replace(N=100, H=64, E=1024, k=8, R=1024), 0.0, 1, "one_tile"),
    (CONFIGS["dsv3"].replace(N=50, H=64, E=64, k=32, R=8), 0.1, 8, "one_tile"),
    (CONFIGS["mixtral"].with_tokens(1), 0.0, 1, "one_tile"),
    # 2..16 tiles: one thread-block cluster, tile counts through distributed shared memory
    (CONFIGS["dsv3"].with_tokens(2048), 0.1, 8, "groups"),
    (CONFIGS["dsv3"].with_tokens(1100), 0.0, 1, "groups"),
    (CONFIGS["dsv3"].with_tokens(129), 0.0, 1, "groups"),
    (CONFIGS["dsv3"].with_tokens(1024), 0.0, 1, "groups"),
    (CONFIGS["dsv3"].with_tokens(700), 0.2, 16, "groups"),
    (CONFIGS["dsv3"].replace(N=1000, H=64, E=1024, k=8, R=1024), 0.05, 1, "groups"),
    (CONFIGS["dsv3"].replace(N=256, H=64, E=64, k=32, R=8), 0.1, 4, "groups"),
    (CONFIGS["mixtral"].with_tokens(1024), 0.0, 1, "groups"),
    (CONFIGS["tiny"].replace(k=1, N=1000), 0.0, 1, "groups"),
    # several clusters and one exchange of their totals
    (CONFIGS["dsv3"].with_tokens(2049), 0.0, 1, "groups"),
    (CONFIGS["dsv3"].with_tokens(4096), 0.1, 8, "groups"),
    (CONFIGS["dsv3"].with_tokens(16384).replace(H=256), 0.0, 1, "groups"),
    (CONFIGS["skew"].with_tokens(16384).replace(H=256), 0.05, 128, "groups"),
    (CONFIGS["mixtral"].replace(H=256), 0.0, 1, "groups"),
    (CONFIGS["long"].replace(H=128), 0.0, 1, "groups"),
    (CONFIGS["dsv3"].replace(N=5000, H=64, E=1024, k=8, R=1024), 0.05, 1, "groups"),
    (CONFIGS["dsv3"].replace(N=3333, H=64, E=64, k=32, R=8), 0.1, 4, "groups"),
], ids=lambda v: f"{v.name}-N{v.N}-E{v.E}-k{v.k}" if hasattr(v, "name") else str(v))
def test_plan_kernels(cfg, frac, align, kind):
    """Routings of at most one tile (N <= 128) take the one-CTA plan kernel and larger ones
    the group kernel (clusters of up to 16 tiles, one exchange between clusters); their plan,
    dispatch and combine match the oracle bit for bit."""
    import moe_expert_shuffling_b200 as ms
    idx, w, x, xs, _ = make_inputs(cfg, 17, y=False)
    if frac > 0:
        idx = drop_some(idx, frac, 3)
    ref = oracle.plan(idx, cfg.E, cfg.R, align=align)
    p = ms.moe_plan_create(cfg.N, cfg.k, cfg.E, cfg.R, align=align)
    p, ti, tw = gpu_plan(idx, w, cfg.E, cfg.R, plan=p)
    assert p.plan_kernels == 1
    assert p.plan_kind == kind
    got = plan_to_host(p)
    for name in ("cnt", "expert_off", "rcnt", "rank_off", "rtok_off", "slot", "src_tok",
                 "src_j", "rtok"):
        assert np.array_equal(got[name], getattr(ref, name)), name
    assert np.array_equal(got["fanout"], ref.fanout)
    assert int(got["err"][0]) == 0
    used = ref.src_tok >= 0
    if cfg.payload == "fp8":
        recv, rs = ms.moe_dispatch(x, p, x_scale=xs)
        want_recv, _ = oracle.dispatch(x.cpu().numpy(), ref.slot, xs.cpu().numpy(), rows=ref.rows)
        got_recv = recv.cpu().numpy()
        assert p.check() == 0
        assert np.array_equal(got_recv[used], want_recv[used])
        return
    recv = ms.moe_dispatch(x, p)
    out = ms.moe_combine(recv, p)
    assert p.check() == 0
    want_recv = oracle.dispatch(bits16(x).view(np.uint8).reshape(cfg.N, -1), ref.slot, rows=ref.rows)
    got_recv = bits16(recv).view(np.uint8).reshape(ref.rows, -1)
    assert np.array_equal(got_recv[used], want_recv[used])
    y_bits = want_recv.view(np.uint16).reshape(ref.rows, cfg.H).copy()
    y_bits[~used] = 0
    assert np.array_equal(bits16(out), oracle.combine(y_bits, ref.slot, w))


@pytest.mark.parametrize("knobs,kind", [
    ({"plan_cluster": 1}, "groups"), ({"plan_cluster": 2}, "groups"),
    ({"plan_cluster": 3}, "groups"), ({"plan_cluster": 8}, "groups"),
    ({"plan_cluster": 16}, "groups"), ({"plan_engine": 3}, "cooperative"),
    ({"plan_engine": 2}, "three"), ({"plan_match": 1}, "groups"), ({"plan_match": 2}, "groups"),
    ({"plan_match": 2, "plan_engine": 3}, "cooperative"),
], ids=lambda v: str(v))
@pytest.mark.parametrize("name,N,frac,align", [("dsv3", 3000, 0.1, 1), ("dsv3", 16384, 0.0, 8),
                                               ("mixtral", 8192, 0.0, 1), ("long", 9000, 0.2, 4),
                                               ("dsv3_k32", 2500, 0.1, 1), ("dsv3_k16", 1100, 0.0, 2)])
def test_plan_engines_agree_with_the_oracle(knobs, kind, name, N, frac, align):
    """Every planner kernel and cluster size gives the oracle's plan bit for bit, including
    repeated calls on one plan (the exchange words are reused) and drops and alignment."""
    import moe_expert_shuffling_b200 as ms
    cfg = CONFIGS[name].with_tokens(N)
    p = ms.moe_plan_create(N, cfg.k, cfg.E, cfg.R, align=align)
    try:
        for k, v in knobs.items():
            ms.moe_tune(k, v)
        for seed in (5, 6):
            idx, w = make_routing(cfg, seed)
            if frac > 0:
                idx = drop_some(idx, frac, seed)
            p, ti, tw = gpu_plan(idx, w, cfg.E, cfg.R, plan=p)
            assert p.plan_kind == kind
            got = plan_to_host(p)
            ref = oracle.plan(idx, cfg.E, cfg.R, align=align)
            for f in ("cnt", "expert_off", "rcnt", "rank_off", "rtok_off", "slot", "src_tok",
                      "src_j", "rtok"):
                assert np.array_equal(got[f], getattr(ref, f)), f
            assert np.array_equal(got["fanout"], ref.fanout)
            assert p.check() == 0
    finally:
        for k in knobs:
            ms.moe_tune(k, 0)
        p.close()


@pytest.mark.parametrize("knobs", [{"combine_max_cw": 4}, {"combine_max_cw": 8},
                                   {"combine_tokens_per_cta": 1}],
                         ids=["4-warps", "8-warps", "1-token-runs"])
@pytest.mark.parametrize("cfg", [CONFIGS["mixtral"].with_tokens(1500),
                                 CONFIGS["long"].replace(N=900, H=512, k=4, E=16, R=16),
                                 CONFIGS["tiny"].replace(k=3, N=333)],
                         ids=lambda c: f"{c.name}-k{c.k}")
def test_small_k_combine_shapes(cfg, knobs):
    """k <= 4 combines with 8 consumer warps (4 KB per row) by default; both chunk widths
    and both orders match the oracle bit for bit."""
    import moe_expert_shuffling_b200 as ms
    idx, w, x, xs, y = make_inputs(cfg, 23)
    ref = oracle.plan(idx, cfg.E, cfg.R)
    try:
        for k, v in knobs.items():
            ms.moe_tune(k, v)
        p, ti, tw = gpu_plan(idx, w, cfg.E, cfg.R)
        out = ms.moe_combine(y, p)
        out_r = ms.moe_combine(y, p, ranked=True)
        assert p.check() == 0
    finally:
        for k in knobs:
            ms.moe_tune(k, 0)
    yb = bits16(y)
    assert np.array_equal(bits16(out), oracle.combine(yb, ref.slot, w))
    assert np.array_equal(bits16(out_r), oracle.combine_ranked(yb, ref.slot, w, idx, cfg.E, cfg.R))


def test_one_plan_reused_across_sizes():
    """One plan object planned again and again with different token counts, so that the
    planner kernel, the number of cluster groups and the exchange generation change from
    call to call (stale arrival words of a larger earlier call stay in memory); every call
    matches the oracle bit for bit."""
    import moe_expert_shuffling_b200 as ms
    cfg = CONFIGS["dsv3"].replace(H=64)
    p = ms.moe_plan_create(16384, cfg.k, cfg.E, cfg.R)
    try:
        for i, N in enumerate((16384, 3000, 129, 16384, 2049, 100, 8192, 16384, 4097)):
            c = cfg.with_tokens(N)
            idx, w = make_routing(c, 40 + i)
            if i % 3 == 1:
                idx = drop_some(idx, 0.1, i)
            p, ti, tw = gpu_plan(idx, w, c.E, c.R, plan=p)
            got = plan_to_host(p)
            ref = oracle.plan(idx, c.E, c.R)
            for f in ("cnt", "expert_off", "rcnt", "rank_off", "rtok_off", "slot", "src_tok",
                      "src_j", "rtok"):
                assert np.array_equal(got[f], getattr(ref, f)), (N, f)
            assert np.array_equal(got["fanout"], ref.fanout)
            assert p.check() == 0
    finally:
        p.close()


@pytest.mark.parametrize("name,N", [("dsv3", 16384), ("dsv3", 3000), ("dsv3", 100),
                                    ("dsv3_k32", 2000), ("mixtral", 4000)])
@pytest.mark.parametrize("engine", [0, 3, 2], ids=["auto", "cooperative", "three"])
def test_plan_without_dedup_lists(name, N, engine):
    """A plan created without the per-rank lists writes everything else bit for bit as the
    oracle does (rcnt and rtok_off included) and leaves the list arrays untouched."""
    import moe_expert_shuffling_b200 as ms
    cfg = CONFIGS[name].with_tokens(N)
    idx, w = make_routing(cfg, 77)
    p = ms.moe_plan_create(N, cfg.k, cfg.E, cfg.R, dedup_lists=False)
    assert not p.dedup_lists
    ms.moe_tune("plan_engine", engine)
    try:
        p, ti, tw = gpu_plan(idx, w, cfg.E, cfg.R, plan=p)   # the lists stay as created: 0
        got = plan_to_host(p)
    finally:
        ms.moe_tune("plan_engine", 0)
    ref = oracle.plan(idx, cfg.E, cfg.R)
    for f in ("cnt", "expert_off", "rcnt", "rank_off", "rtok_off", "slot", "src_tok", "src_j"):
        assert np.array_equal(got[f], getattr(ref, f)), f
    assert not got["rtok"].any() and not got["fanout"].any()
    assert p.check() == 0
    p.close()


@pytest.mark.parametrize("knobs", [{}, {"dispatch_split_units": 1, "combine_split": 1},
                                   {"dispatch_split_units": 100000, "combine_split": 7},
                                   {"combine_split": 2}],
                         ids=["auto", "off", "finest", "two"])
@pytest.mark.parametrize("cfg", [CONFIGS["dsv3"].with_tokens(16), CONFIGS["dsv3"].with_tokens(128),
                                 CONFIGS["dsv3"].with_tokens(300),
                                 CONFIGS["long"].with_tokens(100),
                                 CONFIGS["mixtral"].with_tokens(64),
                                 CONFIGS["dsv3_k32"].with_tokens(50)],
                         ids=lambda c: f"{c.name}-N{c.N}")
def test_small_batch_splits(cfg, knobs):
    """Decode-sized batches cut rows into smaller dispatch chunks and share a token's column
    chunks among several combine CTAs; every split gives the oracle's bytes and bits."""
    import moe_expert_shuffling_b200 as ms
    idx, w, x, xs, y = make_inputs(cfg, 51)
    try:
        for k, v in knobs.items():
            ms.moe_tune(k, v)
        p, ti, tw = gpu_plan(idx, w, cfg.E, cfg.R)
        if cfg.payload == "fp8":
            recv, rs = ms.moe_dispatch(x, p, x_scale=xs)
        else:
            recv, rs = ms.moe_dispatch(x, p), None
        out = ms.moe_combine(y, p)
        out_r = ms.moe_combine(y, p, ranked=True)
        assert p.check() == 0
    finally:
        for k in knobs:
            ms.moe_tune(k, 0)
    ref = oracle.plan(idx, cfg.E, cfg.R)
    if cfg.payload == "fp8":
        want, want_rs = oracle.dispatch(x.cpu().numpy(), ref.slot, xs.cpu().numpy())
        assert np.array_equal(recv.cpu().numpy(), want)
        assert np.array_equal(rs.cpu().numpy().view(np.uint8), want_rs)
    else:
        want = oracle.dispatch(bits16(x).view(np.uint8).reshape(cfg.N, -1), ref.slot)
        assert np.array_equal(bits16(recv).view(np.uint8).reshape(cfg.N * cfg.k, -1), want)
    yb = bits16(y)
    assert np.array_equal(bits16(out), oracle.combine(yb, ref.slot, w))
    assert np.array_equal(bits16(out_r), oracle.combine_ranked(yb, ref.slot, w, idx, cfg.E, cfg.R))
