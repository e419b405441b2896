"""Host-side logic of bench.py (no GPU): the algorithmic byte counts behind the metric,
the per-kernel statistics, the L2 statement, and the DRAM-traffic lookup."""

import json
import os

import pytest

import bench
from workloads import CONFIGS


# Algorithmic bytes per step: each x row read once, each receive row written once, each y
# row read once, each out row written once, plus slots (and weights for combine).  The
# expected values are the formulas worked by hand for each configuration:
#   dispatch = N*Hb + N*k*Hb + 4*N*k,   Hb = 2H (bf16) or H + 4H/128 (fp8 + scales)
#   combine  = 2*N*k*H + 2*N*H + 8*N*k
@pytest.mark.parametrize("name,dispatch,combine", [
    ("tiny", 197_632, 198_656),
    ("mixtral", 201_392_128, 201_457_664),
    ("dsv3", 2_114_453_504, 2_114_977_792),
    ("skew", 2_114_453_504, 2_114_977_792),
    ("long", 1_939_341_312, 3_761_242_112),
])
def test_algorithmic_bytes(name, dispatch, combine):
    cfg = CONFIGS[name]
    assert bench.dispatch_bytes(cfg) == dispatch
    assert bench.combine_bytes(cfg) == combine


def test_bytes_per_token_and_dropped_entries():
    cfg = CONFIGS["dsv3"]
    assert bench.dispatch_bytes(cfg, N=1) == 129_056
    assert bench.combine_bytes(cfg, N=1) == 129_088
    # a dropped entry moves no row: only the slots are still read
    full = bench.dispatch_bytes(cfg)
    fewer = bench.dispatch_bytes(cfg, entries=cfg.N * cfg.k - 10)
    assert full - fewer == 10 * cfg.row_bytes
    assert bench.combine_bytes(cfg) - bench.combine_bytes(cfg, entries=cfg.N * cfg.k - 10) == 10 * 2 * cfg.H


def test_job_throughput_counts_every_rank():
    # 1 GB per rank-step, 10 steps, 4 ranks, slowest rank 8 ms -> 5000 GB/s
    assert bench.job_throughput(10**9, 10, 4, 8.0) == pytest.approx(5000.0)


def test_pct_stats():
    ms = [i / 1000.0 for i in range(1, 102)]  # 1..101 us
    st = bench.pct_stats(ms)
    assert st["n"] == 101
    assert st["median"] == pytest.approx(51.0)
    assert st["p10"] == pytest.approx(11.0)
    assert st["p90"] == pytest.approx(91.0)


def test_kernel_split():
    d = {"plan": 1, "dispatch": 2, "combine": 3, "dispatch_combine": 4}
    assert bench.kernel_split(d, False) == {"plan": 1, "dispatch": 2, "combine": 3}
    assert bench.kernel_split(d, True) == {"plan": 1, "dispatch_combine": 4}
    assert bench.kernel_split({"plan": 1, "dispatch": 2, "combine": 0}, True) == {
        "plan": 1, "dispatch_combine": 2}


def test_l2_note_states_sizes():
    assert "every buffer of the step is larger than the 126 MB L2" in bench.l2_note(CONFIGS["dsv3"])
    note = bench.l2_note(CONFIGS["mixtral"])
    assert "x, out fit in the 126 MB L2" in note and "256 MB" in note


def test_kernel_traffic_lookup(tmp_path, monkeypatch):
    src = tmp_path / "k.cu"
    src.write_text("int f() { return 1; }  // a kernel\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    (tmp_path / "profiles").mkdir()
    rec = {"dispatch_bulk_kernel": {"bytes_per_unit": 100.0, "unit": "token",
                                    "shape": {"H": 7168, "k": 8, "payload": "bf16"},
                                    "sources": ["k.cu"],
                                    "sources_code_sha256": bench.code_digest(["k.cu"])}}
    (tmp_path / "profiles" / "dram_traffic.json").write_text(json.dumps(rec))
    cfg = CONFIGS["dsv3"]
    assert bench.kernel_traffic("dispatch_bulk_kernel", cfg) == 100.0 * cfg.N
    assert bench.kernel_traffic("dispatch_bulk_kernel", cfg, dropped=True) is None
    assert bench.kernel_traffic("dispatch_bulk_kernel", CONFIGS["long"]) is None   # other shape
    assert bench.kernel_traffic("combine_bulk_kernel", cfg) is None                # not captured
    src.write_text("/* reworded */ int f()\n{\n    return 1;  // the same code\n}\n")
    assert bench.kernel_traffic("dispatch_bulk_kernel", cfg) == 100.0 * cfg.N    # comments only
    src.write_text("int f() { return 2; }\n")
    assert bench.kernel_traffic("dispatch_bulk_kernel", cfg) is None               # stale


def test_measured_peak_falls_back(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_hbm_peak() == (bench.FALLBACK_HBM_GBS, "fallback")
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6000.5}))
    assert bench.measured_hbm_peak() == (6000.5, "measured")


def test_step_traffic_lookup(tmp_path, monkeypatch):
    """The whole-step DRAM figure comes from a step capture of the same shape and variant,
    against the step's algorithmic bytes; variants that change the traffic get none."""
    src = tmp_path / "k.cu"
    src.write_text("int f() { return 1; }\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    (tmp_path / "profiles").mkdir()
    shape = {"H": 7168, "k": 8, "payload": "bf16"}
    rec = {key: {"bytes_per_unit": v, "unit": "token", "shape": shape, "sources": ["k.cu"],
                 "sources_code_sha256": bench.code_digest(["k.cu"])}
           for key, v in (("step_dsv3", 260000.0), ("step_dsv3_fused", 258000.0))}
    (tmp_path / "profiles" / "dram_traffic.json").write_text(json.dumps(rec))
    cfg = CONFIGS["dsv3"]
    alg = bench.dispatch_bytes(cfg) + bench.combine_bytes(cfg) + bench.plan_bytes(cfg)
    t = bench.step_traffic(cfg, False, alg)
    assert t["dram_bytes"] == round(260000.0 * cfg.N) and t["algorithmic_bytes"] == alg
    assert t["ratio"] == round(260000.0 * cfg.N / alg, 4)
    assert bench.step_traffic(cfg, True, alg)["dram_bytes"] == round(258000.0 * cfg.N)
    assert bench.step_traffic(cfg, False, alg, dropped=True) is None
    assert bench.step_traffic(cfg, False, alg, aligned=True) is None
    assert bench.step_traffic(cfg, False, alg, ranked=True) is None
    assert bench.step_traffic(CONFIGS["skew"], False, alg) is None   # not captured
