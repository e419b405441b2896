"""Shared helpers for the parity tests: run the CUDA path (through the binding, which
calls the C ABI) and the CPU oracle on the same seeded inputs and compare."""

from __future__ import annotations

import numpy as np
import torch

import oracle
from workloads import Config, make_payload_x, make_payload_y, make_routing

PLAN_FIELDS = ("cnt", "expert_off", "rcnt", "rank_off", "rtok_off", "src_tok", "src_j", "rtok")


def bits16(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32)


def gpu_plan(idx: np.ndarray, w: np.ndarray, E: int, R: int, plan=None):
    import moe_expert_shuffling_b200 as ms
    ti = torch.from_numpy(np.ascontiguousarray(idx)).cuda()
    tw = torch.from_numpy(np.ascontiguousarray(w)).cuda()
    p = ms.moe_plan(ti, tw, E, R, plan=plan)
    return p, ti, tw


def plan_to_host(p) -> dict[str, np.ndarray]:
    a = p.arrays()
    out = {k: v.cpu().numpy() for k, v in a.items()}
    out["fanout"] = out["fanout"].view(np.uint32)
    out["err"] = out["err"].view(np.uint32)
    return out


def assert_plan_equal(got: dict, ref: "oracle.Plan"):
    for name in PLAN_FIELDS:
        g, r = got[name], getattr(ref, name)
        assert g.shape == r.shape, (name, g.shape, r.shape)
        if not np.array_equal(g, r):
            bad = np.nonzero(g.ravel() != r.ravel())[0][:5]
            raise AssertionError(f"{name} differs at {bad}: gpu {g.ravel()[bad]} oracle {r.ravel()[bad]}")
    assert np.array_equal(got["slot"], ref.slot)
    assert np.array_equal(got["fanout"], ref.fanout)
    assert int(got["err"][0]) == 0


def combine_tolerance(got_bits: np.ndarray, ref_bits: np.ndarray):
    """Graded bar: <= 1 bf16 ulp per element, max abs <= 1e-2, max rel <= 8e-3."""
    g = bits_to_f32(got_bits).astype(np.float64)
    r = bits_to_f32(ref_bits).astype(np.float64)
    # ulp distance on the monotone integer line of bf16 bit patterns
    def ordered(b):
        b = b.astype(np.int32)
        return np.where(b & 0x8000, 0x8000 - (b & 0x7FFF), 0x8000 + (b & 0x7FFF))
    ulps = np.abs(ordered(got_bits) - ordered(ref_bits))
    d = np.abs(g - r)
    rel = d / np.maximum(np.abs(r), 2.0 ** -126)
    return int(ulps.max(initial=0)), float(d.max(initial=0.0)), float(rel.max(initial=0.0))


def assert_combine_close(got_bits, ref_bits):
    ulp, ab, rel = combine_tolerance(got_bits, ref_bits)
    assert ulp <= 1 and ab <= 1e-2 and rel <= 8e-3, (ulp, ab, rel)


def make_inputs(cfg: Config, seed: int, device="cuda", y=True):
    idx, w = make_routing(cfg, seed)
    x, xs = make_payload_x(cfg, seed, device)
    yy = make_payload_y(cfg.replace(y="normal"), seed, device) if y else None
    return idx, w, x, xs, yy
