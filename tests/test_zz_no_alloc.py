"""moe_plan_noalloc: the planner for callers that may not allocate device memory.

Some callers of this library cannot call cudaMalloc: a process whose own allocator has
reserved the GPU's memory and does not let libraries allocate behind its back, or a
latency-critical loop that cannot take an allocation's device-wide synchronisation.
moe_plan_noalloc serves them by writing the plan into caller-owned arrays and keeping
its scratch in a fixed array the library declares in device memory.

The test calls it through the C ABI twice in a row (different routings, so the second
call runs on top of the scratch contents the first one left) and checks that every
output matches moe_plan's bit for bit.  This file is collected last on purpose.
"""

import ctypes

import numpy as np
import pytest
import torch

from workloads import CONFIGS, make_routing

pytestmark = pytest.mark.gpu

FIELDS = ("cnt", "expert_off", "rcnt", "rank_off", "rtok_off", "slot", "src_tok", "src_j",
          "rtok", "fanout", "err")


def _lib():
    import moe_expert_shuffling_b200 as ms
    lib = ctypes.CDLL(ms.lib_path())
    vp = ctypes.c_void_p
    i32 = ctypes.c_int32
    lib.moe_plan_noalloc.restype = ctypes.c_int
    lib.moe_plan_noalloc.argtypes = [vp, i32, i32, i32, i32] + [vp] * 11 + [vp]
    lib.moe_last_error.restype = ctypes.c_char_p
    return lib


def _noalloc_plan(lib, idx: torch.Tensor, E: int, R: int, stream):
    N, k = idx.shape
    dev = idx.device
    n_dedup = N * min(k, R)

    def buf(n):
        return torch.full((max(n, 1),), -7, dtype=torch.int32, device=dev)

    out = {"cnt": buf(E), "expert_off": buf(E + 1), "rcnt": buf(R), "rank_off": buf(R + 1),
           "rtok_off": buf(R + 1), "slot": buf(N * k), "src_tok": buf(N * k),
           "src_j": buf(N * k), "rtok": buf(n_dedup), "fanout": buf(n_dedup), "err": buf(1)}
    st = lib.moe_plan_noalloc(idx.data_ptr(), N, k, E, R,
                              *[out[f].data_ptr() for f in FIELDS], stream.cuda_stream)
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


def _same(noalloc: dict, ref: dict, N: int, k: int):
    n_dedup = int(ref["rtok_off"][-1].item())
    for f in FIELDS:
        got = noalloc[f]
        want = ref[f].reshape(-1)
        n = {"slot": N * k, "src_tok": N * k, "src_j": N * k, "rtok": n_dedup,
             "fanout": n_dedup}.get(f, want.numel())
        assert torch.equal(got[:n].cpu(), want[:n].cpu()), f


@pytest.mark.parametrize("name,N,seeds", [("dsv3", 3000, (0, 1)), ("long", 5000, (2, 3)),
                                          ("tiny", 128, (4, 5))])
def test_noalloc_matches_existing_plan_twice(name, N, seeds):
    lib = _lib()
    cfg = CONFIGS[name].with_tokens(N)
    stream = torch.cuda.current_stream()
    for seed in seeds:                       # two calls in a row on the shared scratch
        idx_h, _ = make_routing(cfg, seed)
        idx = torch.from_numpy(idx_h).cuda()
        got = _noalloc_plan(lib, idx, cfg.E, cfg.R, stream)
        torch.cuda.synchronize()
        ref = _existing_plan(idx, cfg.E, cfg.R)
        _same(got, ref, cfg.N, cfg.k)
        assert int(got["err"][0].item()) == 0


def test_noalloc_rejects_more_tokens_than_its_scratch_holds():
    """The size limit is checked on the host before anything else; no array is passed,
    so even a broken check could not launch a kernel (the missing arrays fail next)."""
    lib = _lib()
    N, k, E, R = 1 << 20, 8, 256, 32       # needs 289 * 8192 words > 262144
    st = lib.moe_plan_noalloc(None, N, k, E, R, *([None] * 11), None)
    assert st == 1
    assert b"scratch" in lib.moe_last_error()
