"""Pins for the oracle's plan (histogram, scan, stable slots, per-rank dedup).

The oracle is checked against things other than itself: a hand-derived fixture built on
the pages' Token A / Token B routing example, a brute-force recount written differently
(pure Python over lists), structural invariants, special cases with known answers and a
closed-form statistic of the uniform routing draw.
"""

import json
import os

import numpy as np
import pytest

import oracle
from workloads import CONFIGS, ZIPF_ALPHA, distinct_rank_expectation, find_zipf_alpha, make_routing

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "token_ab_example.json")
GOLDEN_DA = os.path.join(os.path.dirname(__file__), "golden", "token_ab_dropped_aligned.json")


def brute_plan(idx, E, R):
    """Per-entry recount: slot = #entries of lower experts + #earlier tokens on the same expert."""
    idx = [list(map(int, row)) for row in idx]
    N = len(idx)
    k = len(idx[0]) if N else 0
    epr = E // R
    slot = [[0] * k for _ in range(N)]
    for t in range(N):
        for j in range(k):
            e = idx[t][j]
            below = sum(1 for row in idx for v in row if v < e)
            earlier = sum(1 for tp in range(t) if e in idx[tp])
            slot[t][j] = below + earlier
    per_rank = []
    for r in range(R):
        lst = []
        for t in range(N):
            m = 0
            for j in range(k):
                if idx[t][j] // epr == r:
                    m |= 1 << j
            if m:
                lst.append((t, m))
        per_rank.append(lst)
    return slot, per_rank


def check_invariants(p, idx, E, R):
    N, k = idx.shape
    epr = E // R
    assert int(p.cnt.sum()) == N * k
    assert p.expert_off[0] == 0 and p.expert_off[-1] == N * k
    assert np.array_equal(np.diff(p.expert_off.astype(np.int64)), p.cnt)
    assert np.array_equal(p.rank_off, p.expert_off[::epr])
    flat = p.slot.ravel()
    # slots are a permutation of [0, N*k)
    assert np.array_equal(np.sort(flat), np.arange(N * k))
    e = idx.ravel()
    assert np.all(p.expert_off[e] <= flat) and np.all(flat < p.expert_off[e + 1])
    # inverse map
    t_of = np.repeat(np.arange(N), k)
    j_of = np.tile(np.arange(k), N)
    assert np.array_equal(p.src_tok[flat], t_of)
    assert np.array_equal(p.src_j[flat], j_of)
    # stable: inside a segment, tokens ascend
    seg_tok = p.src_tok
    for ee in range(E):
        s = seg_tok[p.expert_off[ee]:p.expert_off[ee + 1]]
        assert np.all(np.diff(s) > 0)
    # dedup: sum rcnt = sum over tokens of distinct ranks
    ranks = np.sort(idx // epr, axis=1)
    distinct = 1 + (np.diff(ranks, axis=1) != 0).sum(axis=1) if k > 1 else np.ones(N, np.int64)
    assert int(p.rcnt.sum()) == int(distinct.sum())
    assert int(p.rcnt.sum()) == oracle.dedup_count(idx, E, R)
    for r in range(R):
        toks = p.rtok[p.rtok_off[r]:p.rtok_off[r + 1]]
        masks = p.fanout[p.rtok_off[r]:p.rtok_off[r + 1]]
        hit = (idx // epr == r)
        want = np.nonzero(hit.any(axis=1))[0]
        assert np.array_equal(toks, want)
        want_m = (hit[want] * (1 << np.arange(k))).sum(axis=1)
        assert np.array_equal(masks, want_m.astype(np.uint32))
        # every column a mask names is an expert of rank r, and its slot lies in rank r
        for t, m in zip(toks[:50], masks[:50]):
            for j in range(k):
                if m >> j & 1:
                    assert p.rank_off[r] <= p.slot[t, j] < p.rank_off[r + 1]


def test_golden_token_ab_example():
    g = json.load(open(GOLDEN))
    idx = np.array(g["topk_idx"], np.int32)
    p = oracle.plan(idx, g["E"], g["R"])
    ex = g["expected"]
    for name in ("cnt", "expert_off", "rank_off", "slot", "src_tok", "src_j", "rcnt",
                 "rtok_off", "rtok", "fanout"):
        assert np.array_equal(getattr(p, name), np.array(ex[name])), name
    assert int(p.cnt.sum()) == ex["entry_moves"]
    assert int(p.rcnt.sum()) == ex["rank_moves"]


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_brute_force_tiny(seed):
    cfg = CONFIGS["tiny"]
    idx, _ = make_routing(cfg, seed)
    p = oracle.plan(idx, cfg.E, cfg.R)
    slot, per_rank = brute_plan(idx, cfg.E, cfg.R)
    assert np.array_equal(p.slot, np.array(slot, np.int32))
    for r in range(cfg.R):
        a, b = p.rtok_off[r], p.rtok_off[r + 1]
        assert [(int(t), int(m)) for t, m in zip(p.rtok[a:b], p.fanout[a:b])] == per_rank[r]
    check_invariants(p, idx, cfg.E, cfg.R)


@pytest.mark.parametrize("name", ["tiny", "mixtral", "dsv3", "skew", "long", "dsv3_k16",
                                  "dsv3_k32"])
def test_invariants_all_configs(name):
    cfg = CONFIGS[name]
    idx, _ = make_routing(cfg, 0)
    p = oracle.plan(idx, cfg.E, cfg.R)
    check_invariants(p, idx, cfg.E, cfg.R)


def test_one_expert_per_rank_dedup_is_identity():
    cfg = CONFIGS["mixtral"]          # R == E
    idx, _ = make_routing(cfg, 1)
    p = oracle.plan(idx, cfg.E, cfg.R)
    assert np.array_equal(p.rcnt, p.cnt)
    assert np.array_equal(p.rtok_off, p.expert_off)
    assert np.array_equal(p.rtok, p.src_tok)
    assert np.array_equal(p.fanout, (1 << p.src_j).astype(np.uint32))


def test_single_rank_moves_every_token_once():
    idx, _ = make_routing(CONFIGS["tiny"].replace(R=1), 2)
    p = oracle.plan(idx, 8, 1)
    assert p.rcnt.tolist() == [idx.shape[0]]
    assert np.array_equal(p.rtok, np.arange(idx.shape[0]))
    assert np.all(p.fanout == (1 << idx.shape[1]) - 1)


def test_top1_is_stable_argsort():
    rng = np.random.default_rng(5)
    idx = rng.integers(0, 16, size=(300, 1)).astype(np.int32)
    p = oracle.plan(idx, 16, 4)
    order = np.argsort(idx[:, 0], kind="stable")
    assert np.array_equal(p.src_tok, order)
    assert np.array_equal(p.slot[order, 0], np.arange(300))


def test_empty_input():
    p = oracle.plan(np.zeros((0, 4), np.int32), 16, 4)
    assert p.cnt.sum() == 0 and p.rcnt.sum() == 0
    assert np.all(p.expert_off == 0) and np.all(p.rtok_off == 0)


@pytest.mark.parametrize("name", ["tiny", "mixtral", "dsv3", "long", "dsv3_k16", "dsv3_k32"])
def test_distinct_rank_closed_form(name):
    """Mean distinct ranks per token matches R * (1 - C(E-E/R, k)/C(E, k)) within 5 s.e."""
    cfg = CONFIGS[name]
    want = distinct_rank_expectation(cfg.E, cfg.k, cfg.R)
    for seed in (0, 1, 2):
        idx, _ = make_routing(cfg, seed)
        epr = cfg.E // cfg.R
        ranks = np.sort(idx // epr, axis=1)
        d = 1 + (np.diff(ranks, axis=1) != 0).sum(axis=1)
        p = oracle.plan(idx, cfg.E, cfg.R)
        assert int(p.rcnt.sum()) == int(d.sum())
        mean = p.rcnt.sum() / cfg.N
        se = max(d.std(), 1e-12) / np.sqrt(cfg.N)
        if d.std() == 0:
            assert mean == pytest.approx(want, abs=1e-12)
        else:
            assert abs(mean - want) < 5 * se, (mean, want, se)


def test_closed_form_values():
    assert distinct_rank_expectation(8, 2, 4) == pytest.approx(13 / 7)
    assert distinct_rank_expectation(8, 2, 8) == pytest.approx(2.0)
    assert distinct_rank_expectation(256, 8, 32) == pytest.approx(7.267, abs=1e-3)
    assert distinct_rank_expectation(64, 6, 16) == pytest.approx(5.316, abs=1e-3)


def test_skew_ratio_on_seed0():
    cfg = CONFIGS["skew"]
    idx, _ = make_routing(cfg, 0)
    p = oracle.plan(idx, cfg.E, cfg.R)
    per_rank = np.diff(p.rank_off.astype(np.int64))
    ratio = per_rank.max() / (cfg.N * cfg.k / cfg.R)
    assert 3.8 <= ratio <= 4.2


def test_zipf_alpha_constant_matches_bisection():
    assert find_zipf_alpha(CONFIGS["skew"], 0) == pytest.approx(ZIPF_ALPHA, rel=1e-6)


@pytest.mark.parametrize("bad", ["dup", "range_hi", "range_neg"])
def test_invalid_routing_rejected(bad):
    idx = np.array([[0, 1], [2, 3]], np.int32)
    if bad == "dup":
        idx[1, 1] = 2
    elif bad == "range_hi":
        idx[0, 0] = 8
    else:
        idx[1, 0] = -2          # -1 would be a dropped entry, not an error
    assert not oracle.validate(idx, 8)
    with pytest.raises(oracle.OracleError):
        oracle.plan(idx, 8, 4)


@pytest.mark.parametrize("E,R,k", [(8, 3, 2), (8, 4, 33), (4, 4, 5), (8, 4, 0)])
def test_invalid_shape_rejected(E, R, k):
    idx = np.zeros((1, max(k, 1)), np.int32)
    if k > 0:
        idx[0] = np.arange(k) % E
    with pytest.raises(oracle.OracleError):
        oracle.plan(idx[:, :max(k, 1)] if k else np.zeros((1, 0), np.int32), E, R)


# ------------------------------------------------- dropped entries and aligned segments
def drop_some(idx, frac, seed):
    rng = np.random.default_rng(seed)
    out = idx.copy()
    out[rng.random(idx.shape) < frac] = -1
    return out


def test_golden_dropped_and_aligned():
    g = json.load(open(GOLDEN_DA))
    p = oracle.plan(np.array(g["topk_idx"], np.int32), g["E"], g["R"], align=g["align"])
    ex = g["expected"]
    assert p.rows == ex["rows"]
    for name in ("cnt", "expert_off", "rank_off", "slot", "src_tok", "src_j", "rcnt",
                 "rtok_off", "rtok", "fanout"):
        assert np.array_equal(getattr(p, name), np.array(ex[name])), name


def check_aligned(p, idx, E, R, align):
    valid = idx >= 0
    assert np.all(p.expert_off % align == 0)
    seg = np.diff(p.expert_off.astype(np.int64))
    assert np.array_equal(seg, (p.cnt + align - 1) // align * align)
    assert int(p.cnt.sum()) == int(valid.sum())
    assert np.all(p.slot[~valid] == -1)
    e = idx[valid]
    s = p.slot[valid]
    assert np.all(p.expert_off[e] <= s) and np.all(s < p.expert_off[e] + p.cnt[e])
    assert len(np.unique(s)) == s.size
    # every row that no entry maps to is marked -1 in the inverse maps
    used = np.zeros(p.rows, bool)
    used[s] = True
    assert np.all(p.src_tok[~used] == -1) and np.all(p.src_j[~used] == -1)
    t_of = np.nonzero(valid)[0]
    assert np.array_equal(p.src_tok[s], t_of)
    # the dedup ignores dropped entries
    epr = E // R
    for r in range(R):
        toks = p.rtok[p.rtok_off[r]:p.rtok_off[r + 1]]
        hit = valid & (np.where(valid, idx, 0) // epr == r)
        assert np.array_equal(toks, np.nonzero(hit.any(axis=1))[0])


@pytest.mark.parametrize("name,frac,align", [("tiny", 0.2, 1), ("tiny", 0.3, 8),
                                             ("dsv3", 0.1, 128), ("long", 0.05, 64),
                                             ("mixtral", 0.5, 16)])
def test_dropped_and_aligned_invariants(name, frac, align):
    cfg = CONFIGS[name].with_tokens(min(CONFIGS[name].N, 2000))
    idx = drop_some(make_routing(cfg, 3)[0], frac, 9)
    p = oracle.plan(idx, cfg.E, cfg.R, align=align)
    check_aligned(p, idx, cfg.E, cfg.R, align)
    # alignment only shifts segments: the rank inside a segment is the tight plan's
    t = oracle.plan(idx, cfg.E, cfg.R, align=1)
    valid = idx >= 0
    e = idx[valid]
    assert np.array_equal(p.slot[valid] - p.expert_off[e], t.slot[valid] - t.expert_off[e])
    assert np.array_equal(p.rtok, t.rtok) and np.array_equal(p.fanout, t.fanout)


def test_brute_force_with_drops():
    cfg = CONFIGS["tiny"]
    idx = drop_some(make_routing(cfg, 4)[0], 0.25, 11)
    p = oracle.plan(idx, cfg.E, cfg.R)
    rows = [[int(v) for v in row] for row in idx]
    for t in range(cfg.N):
        for j in range(cfg.k):
            e = rows[t][j]
            if e < 0:
                assert p.slot[t, j] == -1
                continue
            below = sum(1 for row in rows for v in row if 0 <= v < e)
            earlier = sum(1 for tp in range(t) if e in rows[tp])
            assert p.slot[t, j] == below + earlier


def test_all_dropped():
    idx = -np.ones((50, 4), np.int32)
    p = oracle.plan(idx, 16, 4, align=8)
    assert p.cnt.sum() == 0 and p.rcnt.sum() == 0 and np.all(p.slot == -1)
    assert np.all(p.expert_off == 0) and np.all(p.src_tok == -1)
