"""Parity of moe_dispatch_combine (dispatch and combine in one persistent launch) with the
CPU oracle's dispatch and combine on the same seeded inputs.

The fused call must give exactly what the two separate calls give: receive rows bit for
bit and the combine's fp32 fma chain (or rank-grouped order) bit for bit -- both when the
combine reads other rows and when it reads the rows the same launch dispatches (y = recv,
per-token ready flags)."""

import numpy as np
import pytest
import torch

import oracle
from tests.shuffle_cases import bits16, gpu_plan, make_inputs
from tests.test_oracle_plan import drop_some
from workloads import CONFIGS

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def always_one_launch():
    """These tests exercise the one-launch kernel at every size (by default calls below
    320 MB run the two kernels back to back)."""
    import moe_expert_shuffling_b200 as ms
    ms.moe_tune("fused_min_kb", 1)
    yield
    ms.moe_tune("fused_min_kb", 0)


def oracle_recv(cfg, x, xs, ref):
    if cfg.payload == "fp8":
        return oracle.dispatch(x.cpu().numpy(), ref.slot, xs.cpu().numpy(), rows=ref.rows)
    return oracle.dispatch(bits16(x).view(np.uint8).reshape(cfg.N, -1), ref.slot, rows=ref.rows), None


def got_recv_bytes(cfg, recv):
    if cfg.payload == "fp8":
        return recv.cpu().numpy()
    return bits16(recv).view(np.uint8).reshape(recv.shape[0], -1)


def oracle_out(y_bits, ref, w, idx, cfg, ranked):
    if ranked:
        return oracle.combine_ranked(y_bits, ref.slot, w, idx, cfg.E, cfg.R)
    return oracle.combine(y_bits, ref.slot, w)


def fused_case(cfg, seed, identity, ranked, align=1, drop=0.0, repeat=1):
    """One plan; fused dispatch of x and combine of y (or of recv itself)."""
    import moe_expert_shuffling_b200 as ms
    idx, w, x, xs, y = make_inputs(cfg, seed, y=not identity)
    if drop > 0:
        idx = drop_some(idx, drop, seed + 7)
    ref = oracle.plan(idx, cfg.E, cfg.R, align=align)
    p = ms.moe_plan_create(cfg.N, cfg.k, cfg.E, cfg.R, align=align)
    p, ti, tw = gpu_plan(idx, w, cfg.E, cfg.R, plan=p)
    if not identity and ref.rows != cfg.N * cfg.k:
        g = torch.Generator(device="cuda")
        g.manual_seed(seed)
        y = torch.randn((ref.rows, cfg.H), generator=g, device="cuda").to(torch.bfloat16)
    want_recv, want_rs = oracle_recv(cfg, x, xs, ref)
    used = ref.src_tok >= 0
    for _ in range(repeat):
        recv = torch.full((p.rows, cfg.H), 0, dtype=x.dtype, device="cuda")
        if cfg.payload == "fp8":
            out, rs = ms.moe_dispatch_combine(x, p, recv, y, p, x_scale=xs, ranked=ranked)
        else:
            out = ms.moe_dispatch_combine(x, p, recv, recv if identity else y, p, ranked=ranked)
        torch.cuda.synchronize()
        assert p.check() == 0
        assert np.array_equal(got_recv_bytes(cfg, recv)[used], want_recv[used])
        if cfg.payload == "fp8":
            assert np.array_equal(rs.cpu().numpy().view(np.uint8)[used], want_rs[used])
        y_bits = (want_recv.view(np.uint16).reshape(ref.rows, cfg.H) if identity else bits16(y))
        if identity:
            y_bits = y_bits.copy()
            y_bits[~used] = 0  # rows no entry maps to are never read
        assert np.array_equal(bits16(out), oracle_out(y_bits, ref, w, idx, cfg, ranked))
    return p


CASES = [
    CONFIGS["tiny"],
    CONFIGS["dsv3"].with_tokens(3000),
    CONFIGS["mixtral"].with_tokens(2500),
    CONFIGS["long"].with_tokens(2000),
    CONFIGS["dsv3_k16"].with_tokens(700),
    CONFIGS["dsv3_k32"].with_tokens(400),
    CONFIGS["tiny"].with_tokens(1),
    CONFIGS["tiny"].replace(N=70, H=20000),             # rows of two dispatch chunks
    CONFIGS["long"].replace(N=300, H=512),              # 16-byte scale rows
    CONFIGS["tiny"].replace(k=1, N=777),
    CONFIGS["mixtral"].replace(N=2000, k=4),            # k <= 4: eight consumer warps
    CONFIGS["long"].replace(N=1000, H=512, k=4, E=16, R=16),
    CONFIGS["tiny"].replace(k=3, N=333),
]


@pytest.mark.parametrize("ranked", [False, True], ids=["chain", "ranked"])
@pytest.mark.parametrize("cfg", CASES, ids=lambda c: f"{c.name}-N{c.N}-H{c.H}-k{c.k}-{c.payload}")
def test_fused_matches_oracle(cfg, ranked):
    fused_case(cfg, 4, identity=False, ranked=ranked)


@pytest.mark.parametrize("ranked", [False, True], ids=["chain", "ranked"])
@pytest.mark.parametrize("cfg", [c for c in CASES if c.payload == "bf16"],
                         ids=lambda c: f"{c.name}-N{c.N}-H{c.H}-k{c.k}")
def test_fused_combines_what_it_dispatches(cfg, ranked):
    """y = recv: each token is combined from the rows the same launch wrote for it."""
    fused_case(cfg, 6, identity=True, ranked=ranked)


@pytest.mark.parametrize("cfg", [CONFIGS["dsv3"], CONFIGS["mixtral"]], ids=["dsv3", "mixtral"])
def test_fused_full_size(cfg):
    fused_case(cfg, 0, identity=False, ranked=False)
    fused_case(cfg, 1, identity=True, ranked=False)


def test_fused_repeated_launches_reuse_the_plan():
    """Work counters and the flag epoch carry over from launch to launch."""
    fused_case(CONFIGS["dsv3"].with_tokens(2000), 8, identity=True, ranked=False, repeat=4)


@pytest.mark.parametrize("name,N,frac,align", [
    ("dsv3", 2000, 0.1, 128), ("mixtral", 1500, 0.5, 16), ("tiny", 300, 0.3, 8),
])
@pytest.mark.parametrize("identity", [False, True], ids=["y", "recv"])
def test_fused_dropped_and_aligned(name, N, frac, align, identity):
    fused_case(CONFIGS[name].with_tokens(N), 9, identity=identity, ranked=False, align=align,
               drop=frac)


@pytest.mark.parametrize("knobs", [
    {"fused_dispatch_share": 1},
    {"fused_dispatch_share": 100},
    {"fused_ctas_per_sm": 1},
    {"fused_dispatch_run": 1, "fused_combine_run": 1},
    {"fused_dispatch_run": 32, "fused_combine_run": 64},
    {"fused_smem_kb": 16},
    {"fused_smem_kb": 200, "fused_ctas_per_sm": 1},
])
@pytest.mark.parametrize("identity", [False, True], ids=["y", "recv"])
def test_fused_launch_configuration_does_not_change_results(knobs, identity):
    import moe_expert_shuffling_b200 as ms
    try:
        for k, v in knobs.items():
            ms.moe_tune(k, v)
        fused_case(CONFIGS["dsv3"].with_tokens(1500), 2, identity=identity, ranked=False)
    finally:
        for k in knobs:
            ms.moe_tune(k, 0)


def test_fused_two_micro_batches():
    """Dispatch of micro-batch 1 while micro-batch 0 combines (two plans), then the tail."""
    import moe_expert_shuffling_b200 as ms
    cfg = CONFIGS["dsv3"].with_tokens(1800)
    idx0, w0, x0, _, _ = make_inputs(cfg, 11, y=False)
    idx1, w1, x1, _, _ = make_inputs(cfg, 12, y=False)
    p0, ti0, tw0 = gpu_plan(idx0, w0, cfg.E, cfg.R)
    p1, ti1, tw1 = gpu_plan(idx1, w1, cfg.E, cfg.R)
    recv0 = ms.moe_dispatch(x0, p0)
    recv1 = torch.empty_like(recv0)
    out0 = ms.moe_dispatch_combine(x1, p1, recv1, recv0, p0)
    out1 = ms.moe_combine(recv1, p1)
    torch.cuda.synchronize()
    assert p0.check() == 0 and p1.check() == 0
    for idx, w, x, recv, out in ((idx0, w0, x0, recv0, out0), (idx1, w1, x1, recv1, out1)):
        ref = oracle.plan(idx, cfg.E, cfg.R)
        want_recv, _ = oracle_recv(cfg, x, None, ref)
        assert np.array_equal(got_recv_bytes(cfg, recv), want_recv)
        y_bits = want_recv.view(np.uint16).reshape(ref.rows, cfg.H)
        assert np.array_equal(bits16(out), oracle.combine(y_bits, ref.slot, w))


def test_fused_one_side_empty():
    import moe_expert_shuffling_b200 as ms
    cfg = CONFIGS["dsv3"].with_tokens(500)
    idx, w, x, _, y = make_inputs(cfg, 3)
    p, ti, tw = gpu_plan(idx, w, cfg.E, cfg.R)
    e_idx = torch.zeros((0, cfg.k), dtype=torch.int32, device="cuda")
    e_w = torch.zeros((0, cfg.k), dtype=torch.float32, device="cuda")
    pe = ms.moe_plan(e_idx, e_w, cfg.E, cfg.R)
    x_e = torch.zeros((0, cfg.H), dtype=torch.bfloat16, device="cuda")
    recv_e = torch.zeros((0, cfg.H), dtype=torch.bfloat16, device="cuda")
    out = ms.moe_dispatch_combine(x_e, pe, recv_e, y, p)          # combine only
    recv = torch.empty((p.rows, cfg.H), dtype=torch.bfloat16, device="cuda")
    out_e = ms.moe_dispatch_combine(x, p, recv, recv_e, pe)       # dispatch only
    torch.cuda.synchronize()
    assert out_e.shape == (0, cfg.H) and p.check() == 0 and pe.check() == 0
    ref = oracle.plan(idx, cfg.E, cfg.R)
    assert np.array_equal(bits16(out), oracle.combine(bits16(y), ref.slot, w))
    want_recv, _ = oracle_recv(cfg, x, None, ref)
    assert np.array_equal(got_recv_bytes(cfg, recv), want_recv)


def test_fused_rejects_unsafe_arguments():
    import moe_expert_shuffling_b200 as ms
    cfg = CONFIGS["tiny"]
    idx, w, x, _, y = make_inputs(cfg, 1)
    p, ti, tw = gpu_plan(idx, w, cfg.E, cfg.R)
    q, tq, twq = gpu_plan(idx, w, cfg.E, cfg.R)
    recv = torch.empty((p.rows + 8, cfg.H), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ms.MoeError):   # y overlaps recv without being the same buffer
        ms.moe_dispatch_combine(x, p, recv[:p.rows], recv[8:], p)
    with pytest.raises(ms.MoeError):   # y == recv laid out by another plan
        ms.moe_dispatch_combine(x, p, recv[:p.rows], recv[:p.rows], q)
    lc = CONFIGS["long"].replace(N=64, H=640)  # 20-byte scale rows
    li, lw, lx, lxs, ly = make_inputs(lc, 1)
    lp, lti, ltw = gpu_plan(li, lw, lc.E, lc.R)
    lrecv = torch.empty((lp.rows, lc.H), dtype=lx.dtype, device="cuda")
    with pytest.raises(ms.MoeError):
        ms.moe_dispatch_combine(lx, lp, lrecv, ly, lp, x_scale=lxs)
    torch.cuda.synchronize()
    assert p.check() == 0


def test_fused_inside_a_cuda_graph():
    """A captured launch replayed several times: the epoch comes from device memory, so
    each replay waits for its own dispatch."""
    import moe_expert_shuffling_b200 as ms
    cfg = CONFIGS["dsv3"].with_tokens(2000)
    idx, w, x, _, _ = make_inputs(cfg, 13, y=False)
    ref = oracle.plan(idx, cfg.E, cfg.R)
    want_recv, _ = oracle_recv(cfg, x, None, ref)
    want_out = oracle.combine(want_recv.view(np.uint16).reshape(ref.rows, cfg.H), ref.slot, w)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        p, ti, tw = gpu_plan(idx, w, cfg.E, cfg.R)
        recv = torch.empty((p.rows, cfg.H), dtype=torch.bfloat16, device="cuda")
        out = torch.empty((cfg.N, cfg.H), dtype=torch.bfloat16, device="cuda")
        ms.moe_dispatch_combine(x, p, recv, recv, p, out=out, stream=s)  # warm-up
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        recv.zero_()
        ms.moe_dispatch_combine(x, p, recv, recv, p, out=out, stream=s)
    for _ in range(3):
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert p.check() == 0
        assert np.array_equal(bits16(out), want_out)


@pytest.mark.parametrize("identity", [False, True], ids=["y", "recv"])
def test_small_calls_run_the_two_kernels_with_the_same_results(identity):
    import moe_expert_shuffling_b200 as ms
    ms.moe_tune("fused_min_kb", 0)  # the default threshold: this call is below it
    fused_case(CONFIGS["mixtral"].with_tokens(300), 19, identity=identity, ranked=False)
    fused_case(CONFIGS["dsv3"].with_tokens(200), 20, identity=identity, ranked=True)


@pytest.mark.parametrize("knobs", [{}, {"combine_max_cw": 4}, {"fused_combine_run": 8},
                                   {"fused_smem_kb": 64, "fused_ctas_per_sm": 3}],
                         ids=["default", "4-warps", "8-token-runs", "64KB-3-per-SM"])
@pytest.mark.parametrize("cfg", [CONFIGS["mixtral"].with_tokens(4000),
                                 CONFIGS["mixtral"].replace(N=3000, k=4),
                                 CONFIGS["mixtral"].replace(N=3000, k=3, H=1024)],
                         ids=lambda c: f"mixtral-N{c.N}-k{c.k}-H{c.H}")
@pytest.mark.parametrize("identity", [False, True], ids=["y", "recv"])
def test_fused_small_k_shapes(cfg, knobs, identity):
    """Mixtral-shaped k = 2, 3, 4: the fused kernel's wide combine shape (and the narrower one
    it replaced) match the oracle bit for bit, in both orders."""
    import moe_expert_shuffling_b200 as ms
    try:
        for k, v in knobs.items():
            ms.moe_tune(k, v)
        fused_case(cfg, 30, identity=identity, ranked=False)
        fused_case(cfg, 31, identity=identity, ranked=True)
    finally:
        for k in knobs:
            ms.moe_tune(k, 0)
