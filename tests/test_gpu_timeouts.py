"""The library's bounded device waits, made to run out on purpose through
moe_wait_selftest: each must give up after about a second, report MOE_ERR_TIMEOUT in the
error word the host reads, and leave the CUDA context usable (a normal plan / dispatch /
combine right after it still matches the oracle)."""

import time

import numpy as np
import pytest
import torch

import oracle
from tests.shuffle_cases import bits16, gpu_plan, make_inputs
from workloads import CONFIGS

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("which", [0, 1, 2, 3],
                         ids=["ready_flag", "mbarrier", "grid_barrier", "group_exchange"])
def test_wait_gives_up_and_reports_timeout(which):
    import moe_expert_shuffling_b200 as ms
    torch.cuda.synchronize()
    t0 = time.monotonic()
    flags = ms.moe_wait_selftest(which)
    elapsed = time.monotonic() - t0
    assert flags == ms.ERR_TIMEOUT
    assert 0.5 < elapsed < 30.0

    # the context still works: small steps (one tile, and several groups of tiles) match the
    # oracle
    for cfg in (CONFIGS["tiny"], CONFIGS["dsv3"].with_tokens(3000).replace(H=256)):
        idx, w, x, _, y = make_inputs(cfg, 2)
        p, ti, tw = gpu_plan(idx, w, cfg.E, cfg.R)
        recv = ms.moe_dispatch(x, p)
        out = ms.moe_combine(y, p)
        torch.cuda.synchronize()
        assert p.check() == 0
        ref = oracle.plan(idx, cfg.E, cfg.R)
        assert np.array_equal(bits16(out), oracle.combine(bits16(y), ref.slot, w))
        assert np.array_equal(bits16(recv).view(np.uint8).reshape(cfg.N * cfg.k, -1),
                              oracle.dispatch(bits16(x).view(np.uint8).reshape(cfg.N, -1),
                                              ref.slot))


def test_selftest_rejects_unknown_wait():
    import moe_expert_shuffling_b200 as ms
    with pytest.raises(ms.MoeError):
        ms.moe_wait_selftest(7)
