"""Throughput of the MoE token shuffle (plan + dispatch + combine) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config dsv3] [--impl ours|reference]

One step = one pass of the whole path over one batch: moe_plan (histogram, scan, stable
slots, per-rank dedup lists), moe_dispatch (token-major -> expert-major rows) and
moe_combine (weighted gather-reduce back to token order), all on inputs resident in HBM.
The metric is effective HBM GB/s over the algorithmic bytes of dispatch + combine
(each x row read once, each receive row written once, each y row read once, each out
row written once, plus slots and weights), also given as % of the HBM roofline and as
tokens/s.  With N > 1 (torchrun) every GPU runs an independent replica of the same
workload (the path has no exchange step), timed on the device; the job value is the sum
of all ranks' bytes over the slowest rank's time.

--impl reference times the CPU oracle (single thread, the machine's host core) on a bounded
token sample of the same workload and prints the same metric.

Variants of the step (each prints the same kind of line): --fused (dispatch and combine in
one moe_dispatch_combine launch), --combine ranked (rank-grouped combine order), --align A
and --drop F (aligned segments, dropped entries), --micro-batches M [--overlap | --fused]
(pipelined micro-batches), --no-graph (host launches instead of graph replay).
--latency N1,N2,... prints per-call latencies at small token counts instead.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from workloads import (  # noqa: E402
    CONFIGS, Config, drop_entries, make_expert_outputs, make_payload_x, make_payload_y,
    make_routing,
)

METRIC = "dispatch+combine effective HBM GB/s and % of B200 roofline; tokens/s"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0


# ----------------------------------------------------------------------------- bytes
def dispatch_bytes(cfg: Config, N: int | None = None, entries: int | None = None) -> int:
    """x rows read once, one receive row written per routed entry, N*k slots read."""
    N = cfg.N if N is None else N
    V = N * cfg.k if entries is None else entries
    return N * cfg.row_bytes + V * cfg.row_bytes + 4 * N * cfg.k


def combine_bytes(cfg: Config, N: int | None = None, entries: int | None = None) -> int:
    """One bf16 row of y read per routed entry, N bf16 out rows written, slots and weights."""
    N = cfg.N if N is None else N
    V = N * cfg.k if entries is None else entries
    return 2 * V * cfg.H + 2 * N * cfg.H + 8 * N * cfg.k


def plan_bytes(cfg: Config, N: int | None = None) -> int:
    """ids read; slot, src_tok, src_j written; dedup lists (at most N*min(k,R)) written."""
    N = cfg.N if N is None else N
    return 4 * N * cfg.k * 4 + 8 * N * min(cfg.k, cfg.R)


L2_BYTES = 126 * 2**20


def l2_note(cfg: Config) -> str:
    """How the timed steps avoid L2 reuse (no flush kernel runs between steps)."""
    mb = lambda b: f"{b / 2**20:.0f} MB"
    bufs = [("x", cfg.N * cfg.row_bytes), ("recv", cfg.N * cfg.k * cfg.row_bytes)]
    if cfg.y != "identity":
        bufs.append(("y", cfg.N * cfg.k * cfg.H * 2))
    bufs.append(("out", cfg.N * cfg.H * 2))
    sizes = ", ".join(f"{n} {mb(b)}" for n, b in bufs)
    small = [n for n, b in bufs if b <= L2_BYTES]
    if not small:
        return f"no flush: every buffer of the step is larger than the 126 MB L2 ({sizes})"
    total = sum(b for _, b in bufs)
    return (f"no flush: {', '.join(small)} fit in the 126 MB L2, but one step touches "
            f"{mb(total)} ({sizes}), {total / L2_BYTES:.1f}x the L2, so little of it "
            "survives to the next step")


def workload_name(cfg: Config) -> str:
    return (f"{cfg.name}: N={cfg.N} H={cfg.H} E={cfg.E} k={cfg.k} R={cfg.R} "
            f"{cfg.payload} routing={cfg.routing} weights={cfg.weights} experts={cfg.y}")


def measured_hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            v = float(json.load(f)["hbm_gbs"])
        return v, "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def code_digest(paths) -> str:
    """SHA-256 of C/C++/CUDA sources with comments and whitespace removed: it changes when
    the code changes, not when a comment does."""
    import re
    h = hashlib.sha256()
    for rel in paths:
        with open(os.path.join(ROOT, rel)) as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)   # block comments
        text = re.sub(r"//[^\n]*", " ", text)                # line comments
        h.update("".join(text.split()).encode())
    return h.hexdigest()


def kernel_traffic(kernel: str, cfg: Config, dropped: bool = False):
    """DRAM bytes per launch from the committed ncu summary: the captured bytes per token
    scaled to this launch's tokens, if the capture was of this row shape, with every entry
    routed, and the kernel's code is unchanged since (comments aside); else None."""
    if dropped:
        return None
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)[kernel]
    except Exception:
        return None
    shape = rec.get("shape", {})
    if (shape.get("H"), shape.get("k"), shape.get("payload")) != (cfg.H, cfg.k, cfg.payload):
        return None
    units = cfg.N
    if code_digest(rec["sources"]) != rec.get("sources_code_sha256"):
        return None
    return rec["bytes_per_unit"] * units


def step_traffic(cfg: Config, fused: bool, algorithmic: int, dropped: bool = False,
                 aligned: bool = False, ranked: bool = False):
    """DRAM bytes of one whole step (plan, dispatch, combine -- or plan and the fused
    launch) from the committed ncu capture of consecutive launches with caches left alone
    (--cache-control none), so that lines one kernel leaves dirty in L2 are counted when
    the next one writes them back; scaled per token to this workload when the capture was
    of this shape and the kernels' code is unchanged.  Against the algorithmic bytes."""
    if dropped or aligned or ranked:
        return None
    key = f"step_{cfg.name}" + ("_fused" if fused else "")
    bpt = kernel_traffic(key, cfg)
    if bpt is None:
        return None
    return {"dram_bytes": round(bpt), "algorithmic_bytes": algorithmic,
            "ratio": round(bpt / algorithmic, 4),
            "source": "profiles/dram_traffic.json: " + key}


def pct_stats(ms_list):
    """median / p10 / p90 of event times given in ms, reported in us."""
    v = sorted(1e3 * t for t in ms_list)
    q = lambda f: v[min(len(v) - 1, int(round(f * (len(v) - 1))))]
    return {"median": round(statistics.median(v), 2), "p10": round(q(0.1), 2),
            "p90": round(q(0.9), 2), "n": len(v)}


def kernel_split(d: dict, fused: bool) -> dict:
    """Per-kernel entries of the line: with --fused the dispatch slot holds the one launch
    that does dispatch and combine."""
    d = dict(d)
    if fused:
        if "dispatch_combine" not in d:
            d["dispatch_combine"] = d["dispatch"]
        d.pop("dispatch", None)
        d.pop("combine", None)
    else:
        d.pop("dispatch_combine", None)
    return d


def flushed_kernel_times(step, stream, dev, iters, names=("plan", "dispatch", "combine")):
    """Each kernel of the step (plan, dispatch, combine) timed alone (CUDA events on the
    launching stream), each launch preceded by an L2 flush.  The flush READS a buffer of twice the L2 size: that
    writes back and evicts whatever the previous kernel left dirty and leaves only clean,
    unrelated lines, so the timed kernel neither hits in L2 nor pays for another's
    write-back."""
    l2 = getattr(torch.cuda.get_device_properties(dev), "L2_cache_size", 0) or L2_BYTES
    with torch.cuda.stream(stream):
        scratch = torch.ones(2 * l2 // 4, dtype=torch.float32, device=dev)
        sink = torch.empty((), dtype=torch.float32, device=dev)
    times = {name: [] for name in names}
    for it in range(iters + 3):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * len(names))]
        with torch.cuda.stream(stream):
            for phase in range(len(names)):
                torch.sum(scratch, dim=0, out=sink)
                ev[2 * phase].record(stream)
                step(phase_only=phase)
                ev[2 * phase + 1].record(stream)
        stream.synchronize()
        if it >= 3:  # warm-up
            for phase, name in enumerate(names):
                times[name].append(ev[2 * phase].elapsed_time(ev[2 * phase + 1]))
    out = {name: pct_stats(t) for name, t in times.items()}
    out["flush"] = f"read of a {2 * l2 >> 20} MB buffer before each launch"
    return out


# ---------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, period_ms: int = 100):
        self.gpu = gpu_index
        self.period = period_ms
        self.proc = None
        self.path = None

    def start(self):
        try:
            import tempfile
            fd, self.path = tempfile.mkstemp(prefix=f"clocks_gpu{self.gpu}_", suffix=".csv")
            self.fh = os.fdopen(fd, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", str(self.period)],
                stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        rows = []
        with open(self.path) as f:
            lines = f.readlines()
        os.unlink(self.path)
        for line in lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, flags in rows for i, v in enumerate(flags)
                          if v.lower().startswith("active")})
        return {"sm_mhz": statistics.median(r[0] for r in rows),
                "sm_max_mhz": max(r[1] for r in rows), "reasons": reasons,
                "samples": len(rows)}


# ------------------------------------------------------------------------------ ours
def dist_init(backend: str, rank: int, world: int, local: int | None = None):
    """Join the process group (no-op for world == 1).  NCCL for GPU ranks, gloo on CPU."""
    if world == 1:
        return
    import datetime

    import torch.distributed as dist
    kw = {}
    if backend == "nccl":
        kw["device_id"] = torch.device("cuda", local)
    dist.init_process_group(backend, rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120), **kw)


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dist_init("nccl", rank, world, local)
    return world, rank, local


def rank_seed(seed: int, rank: int) -> int:
    """Each rank runs an independent replica on its own seeded batch."""
    return seed + rank


def max_over_ranks(v: float, world: int) -> float:
    """Slowest rank's value (device timing is per rank; the job ends with the last one)."""
    if world == 1:
        return v
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(bytes_per_rank_step: int, steps: int, world: int, max_ms: float) -> float:
    """Whole-job GB/s: every rank's bytes over the slowest rank's time."""
    return bytes_per_rank_step * steps * world / (max_ms * 1e-3) / 1e9


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def apply_tuning(args):
    """--tune KNOB=VALUE: launch parameters of the library (speed only, never results)."""
    import moe_expert_shuffling_b200 as ms
    for t in args.tune:
        knob, value = t.split("=")
        ms.moe_tune(knob, int(value))


def plan_cost_in_step(step, stream, step_ms: float, args) -> dict:
    """What the plan adds to a graph-replayed step: the same replays of a graph holding only
    dispatch and combine (on the plan already built), against the timed step.  The per-kernel
    event timings launch each kernel from the host between two events, so their plan figure
    is mostly launch latency; this one is measured the way `value` is."""
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        step(phase_only=1)
        if not args.fused:
            step(phase_only=2)
    stream.synchronize()
    n = max(10, min(args.steps, 500))
    with torch.cuda.stream(stream):
        graph.replay()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n):
            graph.replay()
        b.record(stream)
    b.synchronize()
    without = a.elapsed_time(b) / n
    del graph
    return {"step_us": round(1e3 * step_ms, 2), "step_without_plan_us": round(1e3 * without, 2),
            "plan_us": round(1e3 * (step_ms - without), 2),
            "note": "graph replays of the whole step against replays of dispatch + combine alone"}


def run_ours(args):
    import moe_expert_shuffling_b200 as ms
    from moe_expert_shuffling_b200 import build as lib_build

    lib_build.build()
    apply_tuning(args)
    world, rank, local = dist_setup(args)
    cfg = CONFIGS[args.config]
    if args.tokens > 0:
        cfg = cfg.with_tokens(args.tokens)
    seed = rank_seed(args.seed, rank)
    dev = torch.device("cuda", local)
    stream = torch.cuda.Stream(device=dev)

    idx_h, w_h = make_routing(cfg, seed)
    if args.drop > 0:
        idx_h = drop_entries(idx_h, args.drop, seed)
    entries = int((idx_h >= 0).sum())
    rows = cfg.N * cfg.k + cfg.E * (args.align - 1)
    with torch.cuda.stream(stream):
        x, xs = make_payload_x(cfg, seed, dev)
        y = (make_payload_y(cfg, seed, dev) if rows == cfg.N * cfg.k
             else make_expert_outputs(rows, cfg.H, seed, dev) if cfg.y != "identity" else None)
        idx = torch.from_numpy(idx_h).to(dev)
        w = torch.from_numpy(w_h).to(dev)
        recv = torch.empty((rows, cfg.H), dtype=x.dtype, device=dev)
        rs = (torch.empty((rows, cfg.H // 128), dtype=torch.float32, device=dev)
              if cfg.payload == "fp8" else None)
        out = torch.empty((cfg.N, cfg.H), dtype=torch.bfloat16, device=dev)
    stream.synchronize()
    identity = y is None
    plan = ms.moe_plan_create(cfg.N, cfg.k, cfg.E, cfg.R, align=args.align,
                              dedup_lists=not args.no_dedup_lists)

    def step(ev=None, phase_only=None):
        """One step: plan, dispatch, combine (phase_only = 0, 1 or 2 runs just that one).
        With --fused: plan, then dispatch and combine in one launch (phase 1)."""
        if ev is not None:
            ev[0].record(stream)
        if phase_only in (None, 0):
            ms.moe_plan(idx, w, cfg.E, cfg.R, plan=plan, stream=stream)
        if ev is not None:
            ev[1].record(stream)
        if args.fused:
            if phase_only in (None, 1):
                ms.moe_dispatch_combine(x, plan, recv, recv if identity else y, plan, out=out,
                                        x_scale=xs, recv_scale=rs,
                                        ranked=args.combine == "ranked", stream=stream)
            if ev is not None:
                ev[2].record(stream)
                ev[3].record(stream)
            return
        if phase_only in (None, 1):
            if rs is not None:
                ms.moe_dispatch(x, plan, recv=recv, x_scale=xs, recv_scale=rs, stream=stream)
            else:
                ms.moe_dispatch(x, plan, recv=recv, stream=stream)
        if ev is not None:
            ev[2].record(stream)
        if phase_only in (None, 2):
            ms.moe_combine(recv if identity else y, plan, out=out, stream=stream,
                           ranked=args.combine == "ranked")
        if ev is not None:
            ev[3].record(stream)

    for _ in range(args.warmup):
        step()
    stream.synchronize()
    if plan.check(stream) != 0:
        raise SystemExit("device reported invalid routing or a timeout")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    graph = None
    if args.graph:
        # One whole step (plan, dispatch, combine) captured once and replayed: no host work
        # per step.  The per-kernel times come from an event-timed pass of the same steps on
        # the same stream just before the timed replays.
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            step()
        stream.synchronize()
        for i in range(min(args.steps, 200)):
            step(evs[i])
        stream.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize(dev)
    if graph is not None:
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            g0.record(stream)
            for _ in range(args.steps):
                graph.replay()
            g1.record(stream)
    else:
        for i in range(args.steps):
            step(evs[i])
    torch.cuda.synchronize(dev)
    barrier(world)
    clk = clocks.stop()
    if graph is not None:
        elapsed_ms = g0.elapsed_time(g1)
        evs = evs[:min(args.steps, 200)]
    else:
        elapsed_ms = evs[0][0].elapsed_time(evs[-1][3])
    plan_cost = plan_cost_in_step(step, stream, elapsed_ms / args.steps, args) if graph else None
    t_plan = [e[0].elapsed_time(e[1]) for e in evs]
    t_disp = [e[1].elapsed_time(e[2]) for e in evs]
    t_comb = [e[2].elapsed_time(e[3]) for e in evs]
    elapsed_ms = max_over_ranks(elapsed_ms, world)
    ms_per_step = elapsed_ms / args.steps

    db, cb = dispatch_bytes(cfg, entries=entries), combine_bytes(cfg, entries=entries)
    value = job_throughput(db + cb, args.steps, world, elapsed_ms)
    tokens_per_s = cfg.N * args.steps * world / (elapsed_ms * 1e-3)
    peak, peak_kind = measured_hbm_peak()
    disp_us = 1e3 * statistics.mean(t_disp)
    comb_us = 1e3 * statistics.mean(t_comb)
    plan_us = 1e3 * statistics.mean(t_plan)
    if args.fused:
        dom, dom_bytes, dom_us = "fused_dispatch_combine_kernel", db + cb, disp_us
    elif disp_us >= comb_us:
        dom, dom_bytes, dom_us = "dispatch_bulk_kernel", db, disp_us
    else:
        dom, dom_bytes, dom_us = "combine_bulk_kernel", cb, comb_us
    achieved = dom_bytes / (dom_us * 1e-6) / 1e9
    # plan (1 cooperative kernel or 3) + dispatch (+ the scale kernel for fp8 scale rows
    # that are not a multiple of 16 bytes) + combine
    launches_per_step = (plan.plan_kernels + 1 + (0 if args.fused else 1) +
                         (1 if cfg.payload == "fp8" and (4 * (cfg.H // 128)) % 16 else 0))

    # dedup counters (informational, read after the timed region): the plan lists one move
    # per (token, destination rank); entries beyond that are fanned out locally
    moves = int(plan.arrays()["rcnt"].sum().item())
    plan_kind = plan.plan_kind
    dedup = {"entries": entries, "moves": moves,
             "moves_per_token": round(moves / cfg.N, 4),
             "redundant_fraction": round(1.0 - moves / max(entries, 1), 4),
             "wire_bytes": moves * cfg.row_bytes}

    # end to end: pinned host inputs -> device, step, result -> pinned host
    e2e = None
    if args.e2e_steps > 0:
        idx_p = torch.from_numpy(idx_h).pin_memory()
        w_p = torch.from_numpy(w_h).pin_memory()
        x_p = x.cpu().pin_memory()
        xs_p = xs.cpu().pin_memory() if xs is not None else None
        y_p = y.cpu().pin_memory() if y is not None else None
        out_p = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in (idx_p, w_p, x_p, xs_p, y_p) if t is not None)
        d2h = out_p.numel() * out_p.element_size()

        def e2e_step():
            with torch.cuda.stream(stream):
                idx.copy_(idx_p, non_blocking=True)
                w.copy_(w_p, non_blocking=True)
                x.copy_(x_p, non_blocking=True)
                if xs_p is not None:
                    xs.copy_(xs_p, non_blocking=True)
                if y_p is not None:
                    y.copy_(y_p, non_blocking=True)
            step()
            with torch.cuda.stream(stream):
                out_p.copy_(out, non_blocking=True)

        e2e_step()
        stream.synchronize()
        barrier(world)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.e2e_steps):
            e2e_step()
        b.record(stream)
        b.synchronize()
        e_ms = max_over_ranks(a.elapsed_time(b), world)
        e2e = {"value": round(job_throughput(db + cb, args.e2e_steps, world, e_ms), 3),
               "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": round(e_ms / args.e2e_steps, 3), "steps": args.e2e_steps}

    # each kernel alone after an L2 flush (outside the timed region)
    flushed = None
    if args.flushed_iters > 0:
        if args.fused:
            flushed = flushed_kernel_times(step, stream, dev, args.flushed_iters,
                                           names=("plan", "dispatch_combine"))
            sizes = (("dispatch_combine", db + cb), ("plan", plan_bytes(cfg)))
        else:
            flushed = flushed_kernel_times(step, stream, dev, args.flushed_iters)
            sizes = (("dispatch", db), ("combine", cb), ("plan", plan_bytes(cfg)))
        for name, nbytes in sizes:
            flushed[name]["gbs_at_median"] = round(nbytes / (flushed[name]["median"] * 1e-6) / 1e9, 1)

    cpu = None
    if rank == 0 and world == 1 and args.cpu_seconds > 0:
        cpu = cpu_baseline(cfg, idx_h, w_h, x, xs, y, recv, args.cpu_seconds)

    plan.close()
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if cfg.payload == "bf16" else "fp8e4m3", "accum_dtype": "f32",
        "data": "synthetic (seeded routing and N(0,1) payload; no traces or weights exist)",
        "config": {"workload": workload_name(cfg)
                   + ("" if args.combine == "chain" else ", combine grouped by rank")
                   + (f", segments aligned to {args.align} rows" if args.align > 1 else "")
                   + (f", {args.drop:.0%} of entries dropped" if args.drop > 0 else "")
                   + (", dispatch and combine in one launch" if args.fused else "")
                   + (", plan without the per-rank lists" if args.no_dedup_lists else "")
                   + "".join(f", {t}" for t in args.tune),
                   "model": f"{cfg.name}-shaped MoE layer shuffle",
                   "global_batch": cfg.N * world, "seq_len": cfg.N, "parallelism": f"replicas{world}",
                   "ep_ranks_logical": cfg.R,
                   "l2": l2_note(cfg),
                   "launch": "CUDA graph of one step, replayed" if args.graph else "stream"},
        "tokens_per_s": round(tokens_per_s, 1),
        "pct_roofline": {"of_nominal_8000": round(100 * value / world / NOMINAL_HBM_GBS, 2),
                         f"of_{peak_kind}_{peak:g}": round(100 * value / world / peak, 2)},
        "kernels_us": kernel_split({"plan": round(plan_us, 2), "dispatch": round(disp_us, 2),
                                    "combine": round(comb_us, 2)}, args.fused),
        "kernels_unflushed_us": kernel_split(
            {"note": "back-to-back steps on one stream, no flush", "plan": pct_stats(t_plan),
             "dispatch": pct_stats(t_disp), "combine": pct_stats(t_comb)}, args.fused),
        "kernels_flushed_us": flushed,
        "plan_in_step_us": plan_cost,
        "kernels_gbs": kernel_split(
            {"dispatch": round(db / (disp_us * 1e-6) / 1e9, 1),
             "combine": round(cb / (max(comb_us, 1e-3) * 1e-6) / 1e9, 1),
             "dispatch_combine": round((db + cb) / (disp_us * 1e-6) / 1e9, 1),
             "plan": round(plan_bytes(cfg) / (plan_us * 1e-6) / 1e9, 1)}, args.fused),
        "roofline": {"bound": "hbm", "kernel": dom, "achieved": round(achieved, 1),
                     "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": round(achieved / peak, 4),
                     "traffic": kernel_traffic(dom, cfg, dropped=args.drop > 0)},
        "step_traffic": step_traffic(cfg, args.fused, db + cb + plan_bytes(cfg),
                                     dropped=args.drop > 0, aligned=args.align > 1,
                                     ranked=args.combine == "ranked"),
        "gpu_launches": launches_per_step * args.steps,
        "plan_kind": plan_kind,
        "dedup": dedup,
        "clocks": clk,
        "e2e": e2e,
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)


def run_micro_batches(args):
    """The batch split into M micro-batches.  Without --overlap they run one after the
    other; with it, dispatch of micro-batch m runs on a second stream while micro-batch
    m-1 combines (concurrent dispatch and combine, ordered by events); with --fused the
    two run in one moe_dispatch_combine launch."""
    import moe_expert_shuffling_b200 as ms
    from moe_expert_shuffling_b200 import build as lib_build

    lib_build.build()
    apply_tuning(args)
    world, rank, local = dist_setup(args)
    cfg = CONFIGS[args.config]
    if args.tokens > 0:
        cfg = cfg.with_tokens(args.tokens)
    if cfg.payload != "bf16" or cfg.y == "identity":
        raise SystemExit("micro-batch mode takes a bf16 workload with independent expert outputs")
    seed = rank_seed(args.seed, rank)
    dev = torch.device("cuda", local)
    sa, sb = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    idx_h, w_h = make_routing(cfg, seed)
    with torch.cuda.stream(sa):
        x, _ = make_payload_x(cfg, seed, dev)
        y = make_payload_y(cfg, seed, dev)
        idx = torch.from_numpy(idx_h).to(dev)
        w = torch.from_numpy(w_h).to(dev)
        out = torch.empty((cfg.N, cfg.H), dtype=torch.bfloat16, device=dev)
    sa.synchronize()
    M = args.micro_batches
    cuts = [cfg.N * m // M for m in range(M + 1)]
    mbs = []
    for m in range(M):
        a, b = cuts[m], cuts[m + 1]
        mbs.append(dict(idx=idx[a:b], w=w[a:b], x=x[a:b], y=y[a * cfg.k:b * cfg.k],
                        out=out[a:b], plan=ms.moe_plan_create(b - a, cfg.k, cfg.E, cfg.R),
                        recv=torch.empty(((b - a) * cfg.k, cfg.H), dtype=x.dtype, device=dev)))

    def step(e0=None, e1=None):
        if e0 is not None:
            e0.record(sa)
        for mb in mbs:
            ms.moe_plan(mb["idx"], mb["w"], cfg.E, cfg.R, plan=mb["plan"], stream=sa)
        ms.moe_dispatch(mbs[0]["x"], mbs[0]["plan"], recv=mbs[0]["recv"], stream=sa)
        for m in range(1, M):
            if args.fused:
                # dispatch of micro-batch m and combine of m-1 in one launch
                ms.moe_dispatch_combine(mbs[m]["x"], mbs[m]["plan"], mbs[m]["recv"],
                                        mbs[m - 1]["y"], mbs[m - 1]["plan"],
                                        out=mbs[m - 1]["out"], stream=sa)
                continue
            if args.overlap:
                ready = torch.cuda.Event()
                ready.record(sa)
                sb.wait_event(ready)
                ms.moe_dispatch(mbs[m]["x"], mbs[m]["plan"], recv=mbs[m]["recv"], stream=sb)
                done = torch.cuda.Event()
                done.record(sb)
            else:
                ms.moe_dispatch(mbs[m]["x"], mbs[m]["plan"], recv=mbs[m]["recv"], stream=sa)
            ms.moe_combine(mbs[m - 1]["y"], mbs[m - 1]["plan"], out=mbs[m - 1]["out"], stream=sa)
            if args.overlap:
                sa.wait_event(done)
        ms.moe_combine(mbs[-1]["y"], mbs[-1]["plan"], out=mbs[-1]["out"], stream=sa)
        if e1 is not None:
            e1.record(sa)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    step(e0, None)
    for _ in range(args.steps - 2):
        step()
    step(None, e1)
    torch.cuda.synchronize(dev)
    barrier(world)
    el = max_over_ranks(e0.elapsed_time(e1), world)
    nbytes = dispatch_bytes(cfg) + combine_bytes(cfg)
    value = job_throughput(nbytes, args.steps, world, el)
    for mb in mbs:
        assert mb["plan"].check(sa) == 0
        mb["plan"].close()
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank != 0:
        return
    print(json.dumps({
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(el / args.steps, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": workload_name(cfg) + f", {M} micro-batches"
                   + (", dispatch of each fused with the previous combine in one launch"
                      if args.fused else
                      ", dispatch of each overlapping the previous combine" if args.overlap
                      else ", one after the other")},
        "pct_roofline": {"of_nominal_8000": round(100 * value / world / NOMINAL_HBM_GBS, 2)},
        "gpu_launches": ((2 * M + 1) if args.fused else (3 * M)) * args.steps,
    }), flush=True)


def run_latency(args):
    """Latency of one step at small token counts (decode-sized batches): each of plan,
    dispatch, combine, dispatch+combine in one call, and the whole step, captured in a CUDA
    graph and replayed (CUDA events around the replays, mean per replay).  One JSON line per
    token count; not the bench line."""
    import moe_expert_shuffling_b200 as ms
    from moe_expert_shuffling_b200 import build as lib_build

    lib_build.build()
    apply_tuning(args)
    dev = torch.device("cuda", 0)
    s = torch.cuda.Stream(device=dev)

    def replay_us(fn, iters, reps=1):
        """µs per call: a graph holding `reps` calls back to back, replayed `iters` times.
        With reps = 1 every call is its own graph launch, so small calls measure how fast
        graphs are launched; with reps = 20 the calls follow one another on the device, as
        in a decode step captured with the rest of a model."""
        with torch.cuda.stream(s):
            for _ in range(args.warmup):
                fn()
        s.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            for _ in range(reps):
                fn()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(s):
            g.replay()
            a.record(s)
            for _ in range(iters):
                g.replay()
            b.record(s)
        b.synchronize()
        del g
        return round(1e3 * a.elapsed_time(b) / (iters * reps), 2)

    for N in (int(v) for v in args.latency.split(",")):
        cfg = CONFIGS[args.config].with_tokens(N)
        idx_h, w_h = make_routing(cfg, args.seed)
        with torch.cuda.stream(s):
            x, xs = make_payload_x(cfg, args.seed, dev)
            y = make_payload_y(cfg.replace(y="normal"), args.seed, dev)
            idx = torch.from_numpy(idx_h).to(dev)
            w = torch.from_numpy(w_h).to(dev)
            plan = ms.moe_plan_create(N, cfg.k, cfg.E, cfg.R)
            ms.moe_plan(idx, w, cfg.E, cfg.R, plan=plan, stream=s)
            recv = torch.empty((plan.rows, cfg.H), dtype=x.dtype, device=dev)
            rs = (torch.empty((plan.rows, cfg.H // 128), dtype=torch.float32, device=dev)
                  if cfg.payload == "fp8" else None)
            out = torch.empty((N, cfg.H), dtype=torch.bfloat16, device=dev)
        s.synchronize()
        kw = dict(x_scale=xs, recv_scale=rs) if cfg.payload == "fp8" else {}

        def pl():
            ms.moe_plan(idx, w, cfg.E, cfg.R, plan=plan, stream=s)

        def dp():
            ms.moe_dispatch(x, plan, recv=recv, stream=s, **kw)

        def cb():
            ms.moe_combine(y, plan, out=out, stream=s)

        def dc():
            ms.moe_dispatch_combine(x, plan, recv, y, plan, out=out, stream=s, **kw)

        it = max(1, args.steps // 20)
        res = {"workload": workload_name(cfg), "tokens": N, "unit": "us",
               "note": "per call, graphs of 20 calls back to back; single_launch: one call per "
                       "graph launch",
               "plan": replay_us(pl, it, 20), "dispatch": replay_us(dp, it, 20),
               "combine": replay_us(cb, it, 20), "dispatch_combine": replay_us(dc, it, 20),
               "step": replay_us(lambda: (pl(), dp(), cb()), it, 20),
               "single_launch": {"plan": replay_us(pl, args.steps),
                                 "step": replay_us(lambda: (pl(), dp(), cb()), args.steps)},
               "plan_kernels": plan.plan_kernels, "plan_kind": plan.plan_kind}
        if plan.check(s) != 0:
            raise SystemExit("device reported invalid routing or a timeout")
        plan.close()
        print(json.dumps(res), flush=True)


# ------------------------------------------------------------------------ CPU oracle
def oracle_sample_step(cfg: Config, idx_h, w_h, x_bytes, xs_bytes, y_bits, n):
    """One oracle plan + dispatch + combine over the first n tokens of the workload."""
    import oracle
    p = oracle.plan(idx_h[:n], cfg.E, cfg.R)
    if xs_bytes is not None:
        recv, _ = oracle.dispatch(x_bytes[:n], p.slot, xs_bytes[:n])
    else:
        recv = oracle.dispatch(x_bytes[:n], p.slot)
    y = recv.view(np.uint16).reshape(n * cfg.k, cfg.H) if y_bits is None else y_bits[:n * cfg.k]
    oracle.combine(y, p.slot, w_h[:n])


def host_payload(cfg: Config, x, xs, y, n_tokens):
    def bits16(t):
        return t.cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    if cfg.payload == "fp8":
        xb = x[:n_tokens].cpu().numpy()
        xsb = xs[:n_tokens].cpu().numpy().view(np.uint8)
    else:
        xb = bits16(x[:n_tokens]).view(np.uint8).reshape(n_tokens, -1)
        xsb = None
    yb = bits16(y[:n_tokens * cfg.k]) if y is not None else None
    return xb, xsb, yb


def cpu_baseline(cfg, idx_h, w_h, x, xs, y, recv, seconds):
    """Time the oracle as it stands on a token sample sized for about `seconds` of work."""
    n_max = min(cfg.N, 4096)
    xb, xsb, yb = host_payload(cfg, x, xs, y, n_max)
    n = min(64, n_max)
    t0 = time.perf_counter()
    oracle_sample_step(cfg, idx_h, w_h, xb, xsb, yb, n)
    dt = time.perf_counter() - t0
    n = int(max(16, min(n_max, n * (seconds / 3) / max(dt, 1e-6))))
    reps, total_t = 0, 0.0
    while total_t < seconds * 0.66 and reps < 50:
        t0 = time.perf_counter()
        oracle_sample_step(cfg, idx_h, w_h, xb, xsb, yb, n)
        total_t += time.perf_counter() - t0
        reps += 1
    gbs = (dispatch_bytes(cfg, n) + combine_bytes(cfg, n)) * reps / total_t / 1e9
    return {"value": round(gbs, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"first {n} of {cfg.N} tokens (same routing and payload), {reps} "
                      f"plan+dispatch+combine passes, {total_t:.1f} s, single-threaded C",
            "all_cores": cpu_baseline_omp(cfg, idx_h, w_h, xb, xsb, yb, n_max, seconds / 2)}


def cpu_baseline_omp(cfg, idx_h, w_h, xb, xsb, yb, n_max, seconds):
    """The same oracle source built with -fopenmp (dispatch and combine token loops on all
    host cores; the plan stays sequential), on the same kind of sample."""
    import oracle
    from oracle import build as oracle_build
    cores = len(os.sched_getaffinity(0))
    with oracle.using_library(oracle_build.build_omp()):
        n = min(256, n_max)
        t0 = time.perf_counter()
        oracle_sample_step(cfg, idx_h, w_h, xb, xsb, yb, n)
        dt = time.perf_counter() - t0
        n = int(max(16, min(n_max, n * (seconds / 3) / max(dt, 1e-6))))
        reps, total_t = 0, 0.0
        while total_t < seconds * 0.66 and reps < 50:
            t0 = time.perf_counter()
            oracle_sample_step(cfg, idx_h, w_h, xb, xsb, yb, n)
            total_t += time.perf_counter() - t0
            reps += 1
    gbs = (dispatch_bytes(cfg, n) + combine_bytes(cfg, n)) * reps / total_t / 1e9
    return {"value": round(gbs, 4), "unit": "GB/s", "cores": cores,
            "kind": "oracle built with -fopenmp",
            "sample": f"first {n} of {cfg.N} tokens, {reps} passes, {total_t:.1f} s, "
                      f"OMP_NUM_THREADS={os.environ.get('OMP_NUM_THREADS', 'unset (all cores)')}"}


def run_reference(args):
    if int(os.environ.get("RANK", "0")) != 0:
        return
    cfg = CONFIGS[args.config]
    if args.tokens > 0:
        cfg = cfg.with_tokens(args.tokens)
    idx_h, w_h = make_routing(cfg, args.seed)
    n_max = min(cfg.N, 4096)
    cfg_s = cfg.with_tokens(n_max)
    x, xs = make_payload_x(cfg_s, args.seed, "cpu")
    y = make_payload_y(cfg_s, args.seed, "cpu")
    xb, xsb, yb = host_payload(cfg_s, x, xs, y, n_max)
    # size the per-step sample so that warmup + steps take about args.ref_seconds
    n = min(64, n_max)
    t0 = time.perf_counter()
    oracle_sample_step(cfg, idx_h, w_h, xb, xsb, yb, n)
    dt = time.perf_counter() - t0
    per_step = args.ref_seconds / max(1, args.steps + args.warmup)
    n = int(max(16, min(n_max, n * per_step / max(dt, 1e-6))))
    for _ in range(args.warmup):
        oracle_sample_step(cfg, idx_h, w_h, xb, xsb, yb, n)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_sample_step(cfg, idx_h, w_h, xb, xsb, yb, n)
    el = time.perf_counter() - t0
    nbytes = dispatch_bytes(cfg, n) + combine_bytes(cfg, n)
    value = nbytes * args.steps / el / 1e9
    sample = (f"first {n} of {cfg.N} tokens per step (same routing; payload drawn on the host), "
              f"single-threaded C oracle")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * el / args.steps, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if cfg.payload == "bf16" else "fp8e4m3", "accum_dtype": "f32",
        "data": "synthetic", "config": {"workload": workload_name(cfg)},
        "tokens_per_s": round(n * args.steps / el, 1),
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--config", default="dsv3", choices=sorted(CONFIGS))
    ap.add_argument("--tokens", type=int, default=0,
                    help="override the workload's token count (small cases for profiling)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--align", type=int, default=1,
                    help="start every expert segment on a multiple of this many rows")
    ap.add_argument("--drop", type=float, default=0.0,
                    help="fraction of routing entries marked dropped (id -1), seeded")
    ap.add_argument("--graph", dest="graph", action="store_true", default=True,
                    help="capture one step in a CUDA graph and replay it (default)")
    ap.add_argument("--no-graph", dest="graph", action="store_false",
                    help="launch every step from the host on a stream instead")
    ap.add_argument("--micro-batches", type=int, default=1,
                    help="split each step's batch into this many micro-batches")
    ap.add_argument("--overlap", action="store_true",
                    help="with micro-batches: dispatch of one overlaps combine of the previous")
    ap.add_argument("--fused", action="store_true",
                    help="dispatch and combine in one launch (moe_dispatch_combine)")
    ap.add_argument("--combine", default="chain", choices=["chain", "ranked"],
                    help="combine order: one fma chain per token, or grouped by rank first")
    ap.add_argument("--no-dedup-lists", action="store_true",
                    help="plans skip the per-rank lists rtok / fanout (MOE_PLAN_NO_DEDUP_LISTS)")
    ap.add_argument("--tune", action="append", default=[], metavar="KNOB=VALUE",
                    help="set a launch parameter (moe_tune; speed only), repeatable")
    ap.add_argument("--flushed-iters", type=int, default=50,
                    help="iterations of each kernel timed alone after an L2 flush (0: skip)")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--ref-seconds", type=float, default=90.0)
    ap.add_argument("--latency", default="",
                    help="comma-separated token counts: print per-step latencies of the "
                         "workload's shape at each (small batches) instead of the bench line")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")

    if args.impl == "reference":
        run_reference(args)
    elif args.latency:
        run_latency(args)
    elif args.micro_batches > 1:
        run_micro_batches(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
