"""The pins must catch plausible mistakes in the oracle.  Each case plants one mistake in a
copy of oracle.c (on the CPU), builds it, runs the pins against it and expects at least one
pin to fail; the unchanged source must pass them all."""

import json
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import oracle
from oracle.build import SRC, build_variant
from tests.test_oracle_dispatch_combine import (
    bf16_bits_of, bits16, bits_to_f32, exact_combine, exact_combine_ranked, fma_chain_at_scale,
    ranked_at_scale,
)
from tests.test_oracle_plan import GOLDEN, GOLDEN_DA, brute_plan, check_aligned, check_invariants, drop_some
from workloads import CONFIGS, make_routing, make_workload

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTANTS = {
    # stable order broken: fill segments with tokens in descending order
    "descending_fill": ("for (int64_t t = 0; t < N; ++t)\n        for (int32_t j = 0; j < k; ++j) {\n            int32_t e = topk_idx[t * k + j];\n            if (e == DROPPED) {",
                        "for (int64_t t = N - 1; t >= 0; --t)\n        for (int32_t j = 0; j < k; ++j) {\n            int32_t e = topk_idx[t * k + j];\n            if (e == DROPPED) {"),
    # inclusive instead of exclusive segment starts
    "inclusive_scan": ("expert_off[e + 1] = expert_off[e] + (cnt[e] + align - 1) / align * align;",
                       "expert_off[e + 1] = expert_off[e] + (cnt[e] + align - 1) / align * align + (e == 0 ? cnt[0] : 0);"),
    # wrong expert -> rank map in the dedup (modulo instead of blocks)
    "rank_modulo": ("return e != DROPPED && e / epr == r;",
                    "return e != DROPPED && (e + 1) / epr == r;"),
    # rank segment starts taken from the wrong expert
    "rank_off_index": ("rank_off[r] = expert_off[r * epr];", "rank_off[r] = expert_off[r];"),
    # inverse map records the token instead of the column
    "src_j_token": ("src_j[s] = j;", "src_j[s] = (int32_t)t;"),
    # dispatch copies a neighbour's row
    "dispatch_neighbour": ("memcpy(recv + s * row_bytes, x + t * row_bytes, (size_t)row_bytes);",
                           "memcpy(recv + s * row_bytes, x + ((t + 1) % N) * row_bytes, (size_t)row_bytes);"),
    # combine sums the columns in reverse order
    "combine_reversed": ("for (int32_t j = 0; j < k; ++j) {\n                int64_t s = slot[t * k + j];\n                if (s < 0)\n                    continue; /* dropped entry contributes nothing */",
                         "for (int32_t j = k - 1; j >= 0; --j) {\n                int64_t s = slot[t * k + j];\n                if (s < 0)\n                    continue; /* dropped entry contributes nothing */"),
    # multiply then add (two roundings) instead of a fused multiply-add
    "combine_mul_add": ("acc = fmaf(w[t * k + j], bf16_to_f32(y[s * H + c]), acc);",
                        "acc = w[t * k + j] * bf16_to_f32(y[s * H + c]) + acc;"),
    # truncation instead of round-to-nearest-even
    "bf16_truncate": ("u += 0x7fffu + lsb;", "u += 0u * lsb;"),
    # rounding ties away from zero instead of to even
    "bf16_ties_away": ("u += 0x7fffu + lsb;", "u += 0x8000u + 0u * lsb;"),
    # rank-grouped combine visits the ranks in descending order
    "ranked_descending": ("for (int32_t r = 0; r < R; ++r) {\n                int any = 0;",
                          "for (int32_t r = R - 1; r >= 0; --r) {\n                int any = 0;"),
    # segments not padded to the requested alignment
    "align_ignored": ("expert_off[e + 1] = expert_off[e] + (cnt[e] + align - 1) / align * align;",
                      "expert_off[e + 1] = expert_off[e] + cnt[e] + 0 * align;"),
    # dropped entries still placed (as expert 0)
    "dropped_placed": ("            if (e == DROPPED) {\n                slot[t * k + j] = -1;\n                continue;\n            }",
                       "            if (e == DROPPED) {\n                e = 0;\n            }"),
    # drops the last expert of each token
    "skip_last_column": ("for (int32_t j = 0; j < k; ++j)\n            if (topk_idx[t * k + j] != DROPPED)\n                cnt[topk_idx[t * k + j]] += 1;",
                         "for (int32_t j = 0; j + 1 < k; ++j)\n            if (topk_idx[t * k + j] != DROPPED)\n                cnt[topk_idx[t * k + j]] += 1;"),
}


def run_pins():
    """Run a compact set of the pins; return the names of those that fail."""
    failures = []

    def pin(name, fn):
        try:
            fn()
        except (AssertionError, oracle.OracleError, IndexError, ValueError):
            failures.append(name)

    def golden():
        g = json.load(open(GOLDEN))
        p = oracle.plan(np.array(g["topk_idx"], np.int32), g["E"], g["R"])
        for name in ("cnt", "expert_off", "rank_off", "slot", "src_tok", "src_j", "rcnt",
                     "rtok_off", "rtok", "fanout"):
            assert np.array_equal(getattr(p, name), np.array(g["expected"][name])), name
        cb = g["combine"]
        y = bf16_bits_of(cb["y_rows"])
        out = oracle.combine(y, p.slot, np.array(cb["tie_weights"], np.float32))
        assert out.tolist() == cb["tie_out_bits"]

    def brute():
        cfg = CONFIGS["tiny"]
        idx, _ = make_routing(cfg, 0)
        p = oracle.plan(idx, cfg.E, cfg.R)
        slot, per_rank = brute_plan(idx, cfg.E, cfg.R)
        assert np.array_equal(p.slot, np.array(slot, np.int32))
        for r in range(cfg.R):
            a, b = p.rtok_off[r], p.rtok_off[r + 1]
            assert [(int(t), int(m)) for t, m in zip(p.rtok[a:b], p.fanout[a:b])] == per_rank[r]

    def invariants():
        cfg = CONFIGS["dsv3"].with_tokens(300)
        idx, _ = make_routing(cfg, 1)
        check_invariants(oracle.plan(idx, cfg.E, cfg.R), idx, cfg.E, cfg.R)

    def dispatch_rows():
        cfg = CONFIGS["tiny"]
        wl = make_workload(cfg, 0, with_y=False)
        p = oracle.plan(wl.topk_idx, cfg.E, cfg.R)
        xb = bits16(wl.x)
        recv = oracle.dispatch(xb.view(np.uint8).reshape(cfg.N, -1), p.slot)
        rows = recv.view(np.uint16).reshape(cfg.N * cfg.k, cfg.H)
        for t in range(cfg.N):
            for j in range(cfg.k):
                assert rows[p.slot[t, j]].tobytes() == xb[t].tobytes()

    def exact():
        cfg = CONFIGS["dsv3"].with_tokens(24).replace(H=64)
        wl = make_workload(cfg, 0)
        p = oracle.plan(wl.topk_idx, cfg.E, cfg.R)
        yb = bits16(wl.y)
        out = bits_to_f32(oracle.combine(yb, p.slot, wl.topk_w))
        from fractions import Fraction
        for (t, c), v in exact_combine(yb, p.slot, wl.topk_w, range(cfg.N), range(cfg.H)).items():
            assert Fraction(float(out[t, c])) == v

    def chain_at_scale():
        cfg = CONFIGS["dsv3"].with_tokens(256)
        idx, w = make_routing(cfg, 4)
        p = oracle.plan(idx, cfg.E, cfg.R)
        from workloads import make_payload_y
        yb = bits16(make_payload_y(cfg, 4))
        assert np.array_equal(oracle.combine(yb, p.slot, w), fma_chain_at_scale(yb, p.slot, w))

    def ranked():
        cfg = CONFIGS["dsv3"].with_tokens(256)
        wl = make_workload(cfg, 8)
        p = oracle.plan(wl.topk_idx, cfg.E, cfg.R)
        yb = bits16(wl.y)
        assert np.array_equal(
            oracle.combine_ranked(yb, p.slot, wl.topk_w, wl.topk_idx, cfg.E, cfg.R),
            ranked_at_scale(yb, p.slot, wl.topk_w, wl.topk_idx, cfg.E, cfg.R))

    def dropped_aligned():
        g = json.load(open(GOLDEN_DA))
        p = oracle.plan(np.array(g["topk_idx"], np.int32), g["E"], g["R"], align=g["align"])
        for name in ("cnt", "expert_off", "slot", "src_tok", "rtok", "fanout"):
            assert np.array_equal(getattr(p, name), np.array(g["expected"][name])), name
        cfg = CONFIGS["dsv3"].with_tokens(400)
        idx = drop_some(make_routing(cfg, 3)[0], 0.1, 9)
        check_aligned(oracle.plan(idx, cfg.E, cfg.R, align=16), idx, cfg.E, cfg.R, 16)

    def rounding():
        vals = np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, 257.0, 259.0, 1.2345], np.float32)
        assert np.array_equal(oracle.f32_to_bf16(vals), bf16_bits_of(vals))

    for name, fn in (("golden", golden), ("brute", brute), ("invariants", invariants),
                     ("dispatch", dispatch_rows), ("exact_combine", exact),
                     ("chain_at_scale", chain_at_scale), ("ranked", ranked),
                     ("dropped_aligned", dropped_aligned),
                     ("rounding", rounding)):
        pin(name, fn)
    return failures


def test_unchanged_oracle_passes_every_pin():
    assert run_pins() == []


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, tmp_path):
    """A mutant may also corrupt memory and crash, which equally shows the mistake; so the
    pins run in a child process and a crash counts as caught."""
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    lib = build_variant(src.replace(old, new), str(tmp_path / f"oracle_{name}.so"))
    code = ("import sys; sys.path.insert(0, %r); import oracle\n"
            "from tests.test_oracle_mutants import run_pins\n"
            "with oracle.using_library(%r):\n"
            "    f = run_pins()\n"
            "print('FAILED_PINS', ','.join(f))\n" % (ROOT, lib))
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=600,
                       cwd=ROOT)
    caught = r.returncode != 0 or "FAILED_PINS " not in r.stdout or \
        r.stdout.split("FAILED_PINS ", 1)[1].strip() != ""
    assert caught, f"no pin caught the planted mistake {name}: {r.stdout[-500:]}"
