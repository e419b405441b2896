"""moe_plan_noalloc: the planner for callers that may not allocate device memory.

Some callers of this library cannot call cudaMalloc: a process whose own allocator has
reserved the GPU's memory and does not let libraries allocate behind its back, or a
latency-critical loop that cannot take an allocation's device-wide synchronisation.
moe_plan_noalloc serves them by writing the plan into caller-owned arrays and keeping
its scratch in a fixed array the library declares in device memory.

Every test calls it through the C ABI.  Parity: two calls in a row (different routings, so
the second call runs on top of the scratch contents the first one left), each compared bit
for bit with the CPU oracle's plan and with moe_plan's output, with and without dropped
entries, and at the largest token counts the fixed scratch array holds.  The defining
property is checked too: after a warm-up call, further calls leave the device's free memory
unchanged.  This file is collected last on purpose.
"""

import ctypes

import numpy as np
import pytest
import torch

import oracle
from tests.test_oracle_plan import drop_some
from workloads import CONFIGS, make_routing

pytestmark = pytest.mark.gpu

FIELDS = ("cnt", "expert_off", "rcnt", "rank_off", "rtok_off", "slot", "src_tok", "src_j",
          "rtok", "fanout", "err")
SCRATCH_WORDS = 262144   # the fixed array: (E + R + 1) * ceil(N / 128) words at most


def _lib():
    import moe_expert_shuffling_b200 as ms
    lib = ctypes.CDLL(ms.lib_path())
    vp = ctypes.c_void_p
    i32 = ctypes.c_int32
    lib.moe_plan_noalloc.restype = ctypes.c_int
    lib.moe_plan_noalloc.argtypes = [vp, i32, i32, i32, i32] + [vp] * 11 + [vp]
    lib.moe_last_error.restype = ctypes.c_char_p
    return lib


def _buffers(N, k, E, R, dev):
    n_dedup = N * min(k, R)

    def buf(n):
        return torch.full((max(n, 1),), -7, dtype=torch.int32, device=dev)

    return {"cnt": buf(E), "expert_off": buf(E + 1), "rcnt": buf(R), "rank_off": buf(R + 1),
            "rtok_off": buf(R + 1), "slot": buf(N * k), "src_tok": buf(N * k),
            "src_j": buf(N * k), "rtok": buf(n_dedup), "fanout": buf(n_dedup), "err": buf(1)}


def _call(lib, idx: torch.Tensor, E: int, R: int, out: dict, stream) -> int:
    N, k = idx.shape
    return lib.moe_plan_noalloc(idx.data_ptr(), N, k, E, R,
                                *[out[f].data_ptr() for f in FIELDS], stream.cuda_stream)


def _noalloc_plan(lib, idx: torch.Tensor, E: int, R: int, stream):
    N, k = idx.shape
    out = _buffers(N, k, E, R, idx.device)
    st = _call(lib, idx, E, R, out, stream)
    assert st == 0, lib.moe_last_error().decode()
    return out


def _existing_plan(idx: torch.Tensor, E: int, R: int):
    import moe_expert_shuffling_b200 as ms
    w = torch.full(idx.shape, 1.0 / idx.shape[1], dtype=torch.float32, device=idx.device)
    p = ms.moe_plan(idx, w, E, R)
    a = {k: v.clone() for k, v in p.arrays().items()}
    torch.cuda.synchronize()
    p.close()
    return a


def _same_as_existing(noalloc: dict, ref: dict, N: int, k: int):
    n_dedup = int(ref["rtok_off"][-1].item())
    for f in FIELDS:
        got = noalloc[f]
        want = ref[f].reshape(-1)
        n = {"slot": N * k, "src_tok": N * k, "src_j": N * k, "rtok": n_dedup,
             "fanout": n_dedup}.get(f, want.numel())
        assert torch.equal(got[:n].cpu(), want[:n].cpu()), f


def _same_as_oracle(noalloc: dict, ref: "oracle.Plan"):
    want = {"cnt": ref.cnt, "expert_off": ref.expert_off, "rcnt": ref.rcnt,
            "rank_off": ref.rank_off, "rtok_off": ref.rtok_off, "slot": ref.slot.reshape(-1),
            "src_tok": ref.src_tok, "src_j": ref.src_j, "rtok": ref.rtok,
            "fanout": ref.fanout.view(np.int32)}
    for f, w in want.items():
        g = noalloc[f][:w.size].cpu().numpy()
        if not np.array_equal(g, w):
            bad = np.nonzero(g != w)[0][:5]
            raise AssertionError(f"{f} differs at {bad}: gpu {g[bad]} oracle {w[bad]}")
    assert int(noalloc["err"][0].item()) == 0     # drops are not errors


@pytest.mark.parametrize("name,N,seeds,drop", [
    ("dsv3", 3000, (0, 1), 0.0), ("long", 5000, (2, 3), 0.0), ("tiny", 128, (4, 5), 0.0),
    ("mixtral", 2000, (6, 7), 0.0), ("dsv3", 2500, (8, 9), 0.1), ("tiny", 300, (10, 11), 0.3),
])
def test_noalloc_matches_oracle_and_existing_plan_twice(name, N, seeds, drop):
    lib = _lib()
    cfg = CONFIGS[name].with_tokens(N)
    stream = torch.cuda.current_stream()
    for seed in seeds:                       # two calls in a row on the shared scratch
        idx_h, _ = make_routing(cfg, seed)
        if drop > 0:
            idx_h = drop_some(idx_h, drop, seed + 100)
        idx = torch.from_numpy(idx_h).cuda()
        got = _noalloc_plan(lib, idx, cfg.E, cfg.R, stream)
        torch.cuda.synchronize()
        _same_as_oracle(got, oracle.plan(idx_h, cfg.E, cfg.R))
        _same_as_existing(got, _existing_plan(idx, cfg.E, cfg.R), cfg.N, cfg.k)


@pytest.mark.parametrize("cfg", [
    # (1024 + 1024 + 1) * 127 tiles = 260223 words
    CONFIGS["dsv3"].replace(N=127 * 128, H=64, E=1024, k=8, R=1024),
    # (256 + 32 + 1) * 907 tiles = 262123 words
    CONFIGS["dsv3"].replace(N=907 * 128, H=64),
], ids=["E1024-R1024-N16256", "dsv3-N116096"])
def test_noalloc_at_the_scratch_limit(cfg):
    """The largest token count the fixed array holds plans correctly, and one tile more is
    rejected on the host with MOE_EINVAL before anything is enqueued."""
    lib = _lib()
    tiles = -(-cfg.N // 128)
    assert (cfg.E + cfg.R + 1) * tiles <= SCRATCH_WORDS < (cfg.E + cfg.R + 1) * (tiles + 1)
    idx_h, _ = make_routing(cfg, 31)
    idx = torch.from_numpy(idx_h).cuda()
    got = _noalloc_plan(lib, idx, cfg.E, cfg.R, torch.cuda.current_stream())
    torch.cuda.synchronize()
    _same_as_oracle(got, oracle.plan(idx_h, cfg.E, cfg.R))
    st = lib.moe_plan_noalloc(None, cfg.N + 1, cfg.k, cfg.E, cfg.R, *([None] * 11), None)
    assert st == 1 and b"scratch" in lib.moe_last_error()


def test_noalloc_rejects_host_memory():
    """A host array (here a CPU tensor's storage) is refused before any kernel launch."""
    lib = _lib()
    cfg = CONFIGS["tiny"]
    idx_h, _ = make_routing(cfg, 0)
    idx = torch.from_numpy(idx_h).cuda()
    out = _buffers(cfg.N, cfg.k, cfg.E, cfg.R, idx.device)
    out["slot"] = torch.full((cfg.N * cfg.k,), -7, dtype=torch.int32)    # host memory
    st = _call(lib, idx, cfg.E, cfg.R, out, torch.cuda.current_stream())
    assert st == 1 and b"host memory" in lib.moe_last_error()
    st = lib.moe_plan_noalloc(torch.from_numpy(idx_h).data_ptr(), cfg.N, cfg.k, cfg.E, cfg.R,
                              *[_buffers(cfg.N, cfg.k, cfg.E, cfg.R, idx.device)[f].data_ptr()
                                for f in FIELDS], None)
    assert st == 1 and b"topk_idx" in lib.moe_last_error()
    torch.cuda.synchronize()
    assert int((out["slot"] != -7).sum()) == 0    # nothing was written to the host array


def test_noalloc_calls_allocate_no_device_memory():
    """After one warm-up call (which may load the library's kernels), repeated calls leave
    the device's free memory exactly where it was."""
    lib = _lib()
    cfg = CONFIGS["dsv3"].with_tokens(4000)
    stream = torch.cuda.current_stream()
    idx_h, _ = make_routing(cfg, 3)
    idx = torch.from_numpy(idx_h).cuda()
    out = _buffers(cfg.N, cfg.k, cfg.E, cfg.R, idx.device)
    assert _call(lib, idx, cfg.E, cfg.R, out, stream) == 0
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for _ in range(5):
        assert _call(lib, idx, cfg.E, cfg.R, out, stream) == 0
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    _same_as_oracle(out, oracle.plan(idx_h, cfg.E, cfg.R))
