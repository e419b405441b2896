"""Pins for the oracle's dispatch (row scatter) and combine (weighted gather-reduce).

Dispatch is pinned by a byte-level brute force and by its invariants (each token row
appears once per selected expert; segments list the expert's tokens in order).  Combine
is pinned by an exact-rational emulation of the fp32 fma chain and bf16 rounding, by the
identity-experts invariant (combine(dispatch(x)) == x when the weights sum to 1), by
k = 1 un-permutation, by one-hot expert outputs, by the float64 error bound and by the
hand-derived ties of the golden example.
"""

import json
import os
from fractions import Fraction
from math import floor

import numpy as np
import pytest
import torch

import oracle
from workloads import CONFIGS, make_payload_x, make_payload_y, make_routing, make_workload

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "token_ab_example.json")


def bits16(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def bf16_bits_of(vals) -> np.ndarray:
    return bits16(torch.tensor(vals, dtype=torch.float32).to(torch.bfloat16))


def bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32)


# ---------------------------------------------------------------- exact rounding helpers
def _round_binary(q: Fraction, frac_bits: int, emin: int) -> Fraction:
    """Round a rational to the nearest binary float with `frac_bits` fraction bits (ties even)."""
    if q == 0:
        return Fraction(0)
    sign = -1 if q < 0 else 1
    a = abs(q)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    e = max(e, emin)
    ulp = Fraction(2) ** (e - frac_bits)
    m = a / ulp
    n = floor(m)
    r = m - n
    if r > Fraction(1, 2) or (r == Fraction(1, 2) and n % 2 == 1):
        n += 1
    return sign * n * ulp


def f32_round(q):
    return _round_binary(q, 23, -126)


def bf16_round(q):
    return _round_binary(q, 7, -126)


def exact_combine_ranked(y_bits, slot, w, idx, E, R, tokens, cols):
    """Rank-grouped order in exact rationals: per rank an fp32 fma chain, then fp32 adds."""
    y = bits_to_f32(y_bits)
    epr = E // R
    out = {}
    for t in tokens:
        for c in cols:
            total = Fraction(0)
            for r in range(R):
                cols_r = [j for j in range(slot.shape[1]) if idx[t, j] // epr == r]
                if not cols_r:
                    continue
                part = Fraction(0)
                for j in cols_r:
                    part = f32_round(Fraction(float(w[t, j])) * Fraction(float(y[slot[t, j], c])) + part)
                total = f32_round(total + part)
            out[(t, c)] = bf16_round(total)
    return out


def exact_combine(y_bits, slot, w, tokens, cols):
    """fp32 fma chain from +0 in column order j = 0..k-1, then bf16 RNE, in exact rationals."""
    y = bits_to_f32(y_bits)
    out = {}
    for t in tokens:
        for c in cols:
            acc = Fraction(0)
            for j in range(slot.shape[1]):
                prod = Fraction(float(w[t, j])) * Fraction(float(y[slot[t, j], c]))
                acc = f32_round(prod + acc)
            out[(t, c)] = bf16_round(acc)
    return out


def fma_chain_at_scale(y_bits, slot, w):
    """Exact fp32 fma chain (then bf16 RNE) for every output, vectorised.

    Each product of an fp32 weight and a bf16 value is exact in float64.  The float64 sum
    with the fp32 accumulator is exact too unless their exponents are far apart; a two-sum
    finds those rare sums, which are then redone with exact rationals, so every step equals
    a single rounding of the exact value to fp32."""
    from fractions import Fraction
    yv = bits_to_f32(y_bits).astype(np.float64)
    N, k = slot.shape
    acc = np.zeros((N, yv.shape[1]), np.float32)
    for j in range(k):
        prod = w[:, j:j + 1].astype(np.float64) * yv[slot[:, j]]
        a64 = acc.astype(np.float64)
        s = prod + a64
        bb = s - prod
        err = (prod - (s - bb)) + (a64 - bb)
        nxt = s.astype(np.float32)
        for t, c in zip(*np.nonzero(err != 0)):
            exact = Fraction(float(prod[t, c])) + Fraction(float(a64[t, c]))
            nxt[t, c] = np.float32(float(f32_round(exact)))
        acc = nxt
    return bf16_bits_of(acc)


def _round32_sum(p64, a64):
    """fp32 rounding of the exact sum of two float64 arrays holding exact values."""
    from fractions import Fraction
    s = p64 + a64
    bb = s - p64
    err = (p64 - (s - bb)) + (a64 - bb)
    out = s.astype(np.float32)
    for i in zip(*np.nonzero(err != 0)):
        out[i] = np.float32(float(f32_round(Fraction(float(p64[i])) + Fraction(float(a64[i])))))
    return out


def ranked_at_scale(y_bits, slot, w, idx, E, R):
    """Exact rank-grouped order for every output: per rank an fp32 fma chain, fp32 adds."""
    yv = bits_to_f32(y_bits).astype(np.float64)
    N, k = slot.shape
    epr = E // R
    out = np.zeros((N, yv.shape[1]), np.float32)
    for t in range(N):
        total = np.zeros(yv.shape[1], np.float32)
        for r in sorted({int(e) // epr for e in idx[t]}):
            part = np.zeros(yv.shape[1], np.float32)
            for j in range(k):
                if idx[t, j] // epr == r:
                    part = _round32_sum(np.float64(w[t, j]) * yv[slot[t, j]], part.astype(np.float64))
            total = _round32_sum(total.astype(np.float64), part.astype(np.float64))
        out[t] = total
    return bf16_bits_of(out)


# --------------------------------------------------------------------------- dispatch
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_dispatch_brute_force_tiny(seed):
    cfg = CONFIGS["tiny"]
    wl = make_workload(cfg, seed, with_y=False)
    p = oracle.plan(wl.topk_idx, cfg.E, cfg.R)
    xb = bits16(wl.x)
    recv = oracle.dispatch(xb.view(np.uint8).reshape(cfg.N, -1), p.slot)
    rows = recv.view(np.uint16).reshape(cfg.N * cfg.k, cfg.H)
    for t in range(cfg.N):
        for j in range(cfg.k):
            assert rows[p.slot[t, j]].tobytes() == xb[t].tobytes()
    # every receive row equals the row of the token that owns it
    assert np.array_equal(rows, xb[p.src_tok])


def test_dispatch_fp8_scales_move_with_rows():
    cfg = CONFIGS["long"].with_tokens(300)
    idx, _ = make_routing(cfg, 0)
    x, xs = make_payload_x(cfg, 0)
    p = oracle.plan(idx, cfg.E, cfg.R)
    recv, rs = oracle.dispatch(x.numpy(), p.slot, xs.numpy())
    assert recv.shape == (cfg.N * cfg.k, cfg.H)
    assert np.array_equal(recv, x.numpy()[p.src_tok])
    assert np.array_equal(rs.view(np.float32), xs.numpy()[p.src_tok])
    # dequantised rows are within fp8 e4m3 precision of N(0,1) draws: |x| <= 448 * scale
    deq = torch.from_numpy(recv[:8].copy()).view(torch.float8_e4m3fn).float()
    sc = torch.from_numpy(rs[:8].view(np.float32).copy())
    assert torch.all(deq.view(8, -1, 128).abs().amax(-1) <= 448.0)
    assert torch.all(sc > 0)


def test_dispatch_segments_hold_each_experts_tokens():
    cfg = CONFIGS["dsv3"].with_tokens(512)
    idx, _ = make_routing(cfg, 1)
    p = oracle.plan(idx, cfg.E, cfg.R)
    x = np.arange(cfg.N, dtype=np.int64).repeat(2).view(np.uint8).reshape(cfg.N, 16)
    recv = oracle.dispatch(x, p.slot)
    owner = recv.view(np.int64)[:, 0]
    for e in range(cfg.E):
        seg = owner[p.expert_off[e]:p.expert_off[e + 1]]
        assert np.array_equal(seg, np.nonzero((idx == e).any(axis=1))[0])


# ---------------------------------------------------------------------------- combine
def test_bf16_rounding_matches_library():
    rng = np.random.default_rng(0)
    vals = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * np.float32(3.0),
        np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 257.0, 259.0, 2 ** -130,
                  -2 ** -133, 0.0, -0.0, 3.0e38, 1e-45], np.float32),
    ])
    got = oracle.f32_to_bf16(vals)
    want = bf16_bits_of(vals)
    assert np.array_equal(got, want)


def test_combine_exact_rational_tiny():
    cfg = CONFIGS["tiny"]
    wl = make_workload(cfg, 0)
    p = oracle.plan(wl.topk_idx, cfg.E, cfg.R)
    yb = bits16(wl.y)
    out = oracle.combine(yb, p.slot, wl.topk_w)
    ref = exact_combine(yb, p.slot, wl.topk_w, range(0, cfg.N, 9), range(0, cfg.H, 7))
    got = bits_to_f32(out)
    for (t, c), v in ref.items():
        assert Fraction(float(got[t, c])) == v, (t, c)


@pytest.mark.parametrize("name,N", [("dsv3", 256), ("long", 128)])
def test_combine_matches_exact_fma_chain_at_scale(name, N):
    """Every output of a few hundred tokens equals the exact fp32-fma-chain result."""
    cfg = CONFIGS[name].with_tokens(N)
    idx, w = make_routing(cfg, 4)
    p = oracle.plan(idx, cfg.E, cfg.R)
    yb = bits16(make_payload_y(cfg.replace(y="normal"), 4))
    assert np.array_equal(oracle.combine(yb, p.slot, w), fma_chain_at_scale(yb, p.slot, w))


def test_ranked_combine_exact_rational():
    cfg = CONFIGS["dsv3"].with_tokens(12).replace(H=48)
    wl = make_workload(cfg, 5)
    p = oracle.plan(wl.topk_idx, cfg.E, cfg.R)
    yb = bits16(wl.y)
    out = bits_to_f32(oracle.combine_ranked(yb, p.slot, wl.topk_w, wl.topk_idx, cfg.E, cfg.R))
    ref = exact_combine_ranked(yb, p.slot, wl.topk_w, wl.topk_idx, cfg.E, cfg.R,
                               range(cfg.N), range(cfg.H))
    for (t, c), v in ref.items():
        assert Fraction(float(out[t, c])) == v, (t, c)


def test_ranked_combine_matches_exact_order_at_scale():
    cfg = CONFIGS["dsv3"].with_tokens(256)
    wl = make_workload(cfg, 8)
    p = oracle.plan(wl.topk_idx, cfg.E, cfg.R)
    yb = bits16(wl.y)
    assert np.array_equal(oracle.combine_ranked(yb, p.slot, wl.topk_w, wl.topk_idx, cfg.E, cfg.R),
                          ranked_at_scale(yb, p.slot, wl.topk_w, wl.topk_idx, cfg.E, cfg.R))


def test_ranked_combine_with_one_rank_is_the_plain_chain():
    cfg = CONFIGS["dsv3"].with_tokens(64).replace(H=128, R=1)
    wl = make_workload(cfg, 6)
    p = oracle.plan(wl.topk_idx, cfg.E, cfg.R)
    yb = bits16(wl.y)
    assert np.array_equal(oracle.combine_ranked(yb, p.slot, wl.topk_w, wl.topk_idx, cfg.E, 1),
                          oracle.combine(yb, p.slot, wl.topk_w))


def test_ranked_combine_differs_from_the_chain_only_by_rounding():
    cfg = CONFIGS["dsv3"].with_tokens(128)
    wl = make_workload(cfg, 7)
    p = oracle.plan(wl.topk_idx, cfg.E, cfg.R)
    yb = bits16(wl.y)
    a = oracle.combine_ranked(yb, p.slot, wl.topk_w, wl.topk_idx, cfg.E, cfg.R)
    b = oracle.combine(yb, p.slot, wl.topk_w)
    exact = oracle.combine_f64(yb, p.slot, wl.topk_w)
    assert not np.array_equal(a, b)          # the order matters somewhere
    fa = bits_to_f32(a).astype(np.float64)
    yv = bits_to_f32(yb).astype(np.float64)
    mag = sum(np.abs(wl.topk_w[:, j:j + 1].astype(np.float64) * yv[p.slot[:, j]])
              for j in range(cfg.k))
    gamma = 2 * cfg.k * 2.0 ** -24 / (1 - 2 * cfg.k * 2.0 ** -24)
    assert np.all(np.abs(fa - exact) <= np.abs(exact) * 2.0 ** -8 + 2.0 ** -134 + 1.01 * gamma * mag)


@pytest.mark.parametrize("name,N", [("dsv3", 96), ("long", 96)])
def test_ranked_identity_experts_return_x(name, N):
    cfg = CONFIGS[name].with_tokens(N).replace(payload="bf16")
    wl = make_workload(cfg, 0, with_y=False)
    p = oracle.plan(wl.topk_idx, cfg.E, cfg.R)
    xb = bits16(wl.x)
    recv = oracle.dispatch(xb.view(np.uint8).reshape(N, -1), p.slot).view(np.uint16).reshape(-1, cfg.H)
    out = oracle.combine_ranked(recv, p.slot, wl.topk_w, wl.topk_idx, cfg.E, cfg.R)
    assert np.array_equal(bits_to_f32(out), bits_to_f32(xb))


def test_combine_golden_ties_and_identity():
    g = json.load(open(GOLDEN))
    idx = np.array(g["topk_idx"], np.int32)
    p = oracle.plan(idx, g["E"], g["R"])
    cb = g["combine"]
    x = bf16_bits_of(cb["x"])
    recv = oracle.dispatch(x.view(np.uint8).reshape(3, -1), p.slot).view(np.uint16).reshape(9, 2)
    out = oracle.combine(recv, p.slot, np.array(cb["identity_weights"], np.float32))
    assert np.array_equal(out, bf16_bits_of(cb["identity_out"]))
    y = bf16_bits_of(cb["y_rows"])
    out2 = oracle.combine(y, p.slot, np.array(cb["tie_weights"], np.float32))
    assert out2.tolist() == cb["tie_out_bits"]
    assert np.array_equal(bits_to_f32(out2), np.array(cb["tie_out"], np.float32))


@pytest.mark.parametrize("name,N", [("tiny", 128), ("mixtral", 256), ("dsv3", 96), ("skew", 96)])
def test_identity_experts_return_x(name, N):
    """combine(dispatch(x)) == x when y = recv and the weights sum to 1 (fp32 within k ulp)."""
    cfg = CONFIGS[name].with_tokens(N)
    wl = make_workload(cfg, 0, with_y=False)
    p = oracle.plan(wl.topk_idx, cfg.E, cfg.R)
    xb = bits16(wl.x)
    recv = oracle.dispatch(xb.view(np.uint8).reshape(N, -1), p.slot).view(np.uint16).reshape(-1, cfg.H)
    out = oracle.combine(recv, p.slot, wl.topk_w)
    assert np.array_equal(bits_to_f32(out), bits_to_f32(xb))


def test_top1_unit_weight_unpermutes():
    cfg = CONFIGS["tiny"].replace(k=1)
    wl = make_workload(cfg, 3)
    p = oracle.plan(wl.topk_idx, cfg.E, cfg.R)
    yb = bits16(wl.y)
    out = oracle.combine(yb, p.slot, np.ones((cfg.N, 1), np.float32))
    assert np.array_equal(out, yb[p.slot[:, 0]])


def test_one_hot_rows_give_weight_columns():
    cfg = CONFIGS["dsv3"].with_tokens(64).replace(H=64)
    idx, w = make_routing(cfg, 2)
    p = oracle.plan(idx, cfg.E, cfg.R)
    y = np.zeros((cfg.N * cfg.k, cfg.H), np.float32)
    # receive row of entry (t, j) is one-hot at column j
    for t in range(cfg.N):
        for j in range(cfg.k):
            y[p.slot[t, j], j] = 1.0
    out = bits_to_f32(oracle.combine(bf16_bits_of(y), p.slot, w))
    assert np.array_equal(out[:, :cfg.k], bits_to_f32(bf16_bits_of(w)))
    assert np.all(out[:, cfg.k:] == 0)


@pytest.mark.parametrize("name,N", [("dsv3", 64), ("long", 64), ("mixtral", 64)])
def test_combine_within_float64_error_bound(name, N):
    """|out - exact| <= half a bf16 ulp of the fp32 chain + gamma_k * sum |w y|."""
    cfg = CONFIGS[name].with_tokens(N)
    idx, w = make_routing(cfg, 1)
    p = oracle.plan(idx, cfg.E, cfg.R)
    yb = bits16(make_payload_y(cfg.replace(y="normal"), 1))
    out = bits_to_f32(oracle.combine(yb, p.slot, w)).astype(np.float64)
    exact = oracle.combine_f64(yb, p.slot, w)
    yv = bits_to_f32(yb).astype(np.float64)
    mag = np.zeros_like(exact)
    for j in range(cfg.k):
        mag += np.abs(w[:, j:j + 1].astype(np.float64) * yv[p.slot[:, j]])
    u = 2.0 ** -24
    gamma = cfg.k * u / (1 - cfg.k * u)
    chain_err = gamma * mag
    half_ulp = np.abs(exact) * 2.0 ** -8 + 2.0 ** -134  # >= half a bf16 ulp (7 fraction bits)
    assert np.all(np.abs(out - exact) <= half_ulp + chain_err * 1.01)


def test_dispatch_and_combine_skip_dropped_entries():
    """A dropped entry gets no row and adds nothing: combine equals the chain over the
    token's remaining columns (computed with k-1 columns by moving the dropped one out)."""
    cfg = CONFIGS["tiny"].replace(k=3)
    wl = make_workload(cfg, 2)
    idx = wl.topk_idx.copy()
    idx[::3, 2] = -1                        # drop the last column of every third token
    p = oracle.plan(idx, cfg.E, cfg.R, align=4)
    xb = bits16(wl.x)
    recv = oracle.dispatch(xb.view(np.uint8).reshape(cfg.N, -1), p.slot, rows=p.rows)
    rows16 = recv.view(np.uint16).reshape(p.rows, cfg.H)
    used = p.src_tok >= 0
    assert np.array_equal(rows16[used], xb[p.src_tok[used]])
    assert not rows16[~used].any()          # rows no entry maps to are left untouched
    y = np.random.default_rng(1).standard_normal((p.rows, cfg.H)).astype(np.float32)
    yb = bf16_bits_of(y)
    out = oracle.combine(yb, p.slot, wl.topk_w)
    # reference: for dropped tokens use only columns 0..1 (a k=2 chain), else all three
    w2 = wl.topk_w.copy()
    sl2 = p.slot.copy()
    keep = idx[:, 2] >= 0
    ref_full = oracle.combine(yb, np.where(sl2 < 0, 0, sl2), w2)
    ref_two = oracle.combine(yb, np.ascontiguousarray(sl2[:, :2]), np.ascontiguousarray(w2[:, :2]))
    assert np.array_equal(out[keep], ref_full[keep])
    assert np.array_equal(out[~keep], ref_two[~keep])


def test_openmp_build_gives_the_same_bytes():
    """The -fopenmp build (used only for the multi-core CPU baseline) must compute exactly
    what the oracle computes: its parallel token loops write disjoint rows."""
    from oracle import build as oracle_build
    cfg = CONFIGS["dsv3"].with_tokens(96)
    idx, w = make_routing(cfg, 3)
    x, _ = make_payload_x(cfg, 3, "cpu")
    y = make_payload_y(cfg, 3, "cpu")
    xb = x.contiguous().view(torch.int16).numpy().view(np.uint8).reshape(cfg.N, -1)
    yb = y.contiguous().view(torch.int16).numpy().view(np.uint16)
    p = oracle.plan(idx, cfg.E, cfg.R)
    recv = oracle.dispatch(xb, p.slot)
    out = oracle.combine(yb, p.slot, w)
    with oracle.using_library(oracle_build.build_omp()):
        recv_omp = oracle.dispatch(xb, p.slot)
        out_omp = oracle.combine(yb, p.slot, w)
    assert np.array_equal(recv, recv_omp)
    assert np.array_equal(out, out_omp)
