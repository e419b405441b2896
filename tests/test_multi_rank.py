"""The benchmark's multi-GPU mode runs one independent replica per rank (the shuffle has
no exchange step on one GPU's logical ranks), times each on its device and reports the
job throughput over the slowest rank.  These tests run that host logic as two gloo ranks
on the CPU, with the oracle standing in for each rank's device work."""

import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import bench
    import oracle
    from workloads import CONFIGS, make_routing

    bench.dist_init("gloo", rank, world)
    try:
        # each rank plans its own seeded batch (a replica), as bench.py does per GPU
        cfg = CONFIGS["tiny"]
        seed = bench.rank_seed(7, rank)
        idx, _ = make_routing(cfg, seed)
        p = oracle.plan(idx, cfg.E, cfg.R)
        moves = int(p.rcnt.sum())
        # per-rank "device time": rank r takes (r + 1) * 10 ms
        local_ms = 10.0 * (rank + 1)
        bench.barrier(world)
        max_ms = bench.max_over_ranks(local_ms, world)
        value = bench.job_throughput(1_000_000, 5, world, max_ms)
        gathered = [None] * world
        dist.all_gather_object(gathered, (seed, moves))
        out.put((rank, max_ms, value, gathered))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_aggregate_like_the_benchmark():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    mp.start_processes(_rank_main, args=(world, _free_port(), q), nprocs=world, join=True,
                       start_method="spawn")
    res = sorted(q.get() for _ in range(world))
    for rank, max_ms, value, gathered in res:
        assert max_ms == pytest.approx(20.0)                       # slowest rank
        assert value == pytest.approx(2 * 1_000_000 * 5 / 0.020 / 1e9)
        assert [g[0] for g in gathered] == [7, 8]                  # independent seeds
    # replicas are independent: each rank's plan matches a single-process run of its seed
    sys.path.insert(0, ROOT)
    import oracle
    from workloads import CONFIGS, make_routing
    cfg = CONFIGS["tiny"]
    for seed, moves in res[0][3]:
        idx, _ = make_routing(cfg, seed)
        assert int(oracle.plan(idx, cfg.E, cfg.R).rcnt.sum()) == moves


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.job_throughput(2_000_000_000, 10, 1, 1000.0) == pytest.approx(20.0)
    assert bench.rank_seed(0, 0) == 0


def test_reference_arm_on_nonzero_rank_prints_nothing():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "3", "--warmup", "3"],
                       capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_reference_arm_prints_one_line():
    import json
    env = dict(os.environ, RANK="0", WORLD_SIZE="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--config", "tiny", "--steps", "3", "--warmup", "3",
                        "--ref-seconds", "2"],
                       capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "GB/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0
    assert np.isfinite(d["ms_per_step"])
