"""Seeded generators for the five shuffle workloads.

Workload shapes follow the pages' workloads: a Mixtral-like top-2 of 8 experts, a
DeepSeek-V3-like top-8 of 256 experts on 32 expert-parallel ranks (the model named in
"Accelerating MoE with Dynamic In-Switch Computing on Multi-GPUs", sections 1 and 7),
the same with skewed expert popularity, and a long-context fp8 case (the FUSCO
summary, Group 2, notes that the shuffle overhead grows with context length).  No real
routing traces exist here; these draws stand in for them.

Recipe (every draw is seeded; nothing depends on the machine):

* routing: iid N(0,1) logits ``z[t, e]`` in float64 from numpy PCG64; the top-k ids
  are the k largest logits, listed by descending logit (ties broken by the lower id).
  Weights are either a softmax over the k selected logits or sigmoid(l)/sum sigmoid(l)
  over them, computed in float64 and stored as float32.
* skewed routing: ``l[t, e] = z[t, e] + alpha * ln p_e`` with
  ``p_e ~ (pi(e) + 1) ** -1.2`` (normalised to sum 1) and ``pi`` a permutation of the
  experts drawn from seed 0.  ``alpha`` is fixed so that, on seed 0, the busiest rank
  receives 4.0 +- 0.2 times the mean number of routed entries.  The same biased logits
  feed the top-k and the weights.
* payload ``x``: iid N(0,1) float32 rounded to bf16; for fp8, each run of 128 columns
  of a row is scaled by ``amax / 448`` and cast to float8 e4m3 (the scale is stored
  as float32 beside the row).
* expert outputs ``y``: iid N(0,1) bf16 rows, one per routed entry; or, for "identity
  experts", the dispatched rows themselves (the caller passes its own dispatch output).

Payload tensors are drawn with torch's generator on the requested device; the same
seed gives different values on CPU and CUDA, so a check that needs the host copy of a
device-drawn tensor copies it back rather than re-drawing it.
"""

from __future__ import annotations

import dataclasses
from dataclasses import dataclass

import numpy as np
import torch

FP8_MAX = 448.0          # largest finite float8 e4m3 value
SCALE_COLS = 128         # columns per fp32 scale for fp8 payloads
ZIPF_S = 1.2
SKEW_TARGET = 4.0

# Found with find_zipf_alpha(CONFIGS["skew"], seed=0); pinned by a CPU test.
ZIPF_ALPHA = 0.5009725093841553


@dataclass(frozen=True)
class Config:
    name: str
    N: int            # tokens
    H: int            # hidden size (elements per row)
    E: int            # experts
    k: int            # experts per token
    R: int            # logical expert-parallel ranks
    payload: str      # "bf16" | "fp8"
    routing: str      # "uniform" | "zipf"
    weights: str      # "softmax" | "sigmoid"
    y: str            # "normal" | "identity"

    @property
    def experts_per_rank(self) -> int:
        return self.E // self.R

    def with_tokens(self, N: int) -> "Config":
        return dataclasses.replace(self, N=N)

    def replace(self, **kw) -> "Config":
        return dataclasses.replace(self, **kw)

    @property
    def row_bytes(self) -> int:
        """Payload bytes of one row, fp8 scales included."""
        if self.payload == "fp8":
            return self.H + 4 * (self.H // SCALE_COLS)
        return 2 * self.H


CONFIGS = {
    "tiny": Config("tiny", N=128, H=256, E=8, k=2, R=4, payload="bf16",
                   routing="uniform", weights="softmax", y="normal"),
    "mixtral": Config("mixtral", N=8192, H=4096, E=8, k=2, R=8, payload="bf16",
                      routing="uniform", weights="softmax", y="identity"),
    "dsv3": Config("dsv3", N=16384, H=7168, E=256, k=8, R=32, payload="bf16",
                   routing="uniform", weights="sigmoid", y="normal"),
    "skew": Config("skew", N=16384, H=7168, E=256, k=8, R=32, payload="bf16",
                   routing="zipf", weights="sigmoid", y="normal"),
    "long": Config("long", N=65536, H=4096, E=64, k=6, R=16, payload="fp8",
                   routing="uniform", weights="softmax", y="normal"),
    # DeepSeek-V3 with wider top-k, the medium and large settings of the DySHARP study
    # (topk 16 and 32; "Accelerating MoE with Dynamic In-Switch Computing", section 7)
    "dsv3_k16": Config("dsv3_k16", N=16384, H=7168, E=256, k=16, R=32, payload="bf16",
                       routing="uniform", weights="sigmoid", y="normal"),
    "dsv3_k32": Config("dsv3_k32", N=16384, H=7168, E=256, k=32, R=32, payload="bf16",
                       routing="uniform", weights="sigmoid", y="normal"),
}


@dataclass
class Workload:
    cfg: Config
    seed: int
    topk_idx: np.ndarray          # int32 [N, k]
    topk_w: np.ndarray            # float32 [N, k]
    x: torch.Tensor               # bf16 [N, H], or uint8 [N, H] holding fp8 e4m3 bytes
    x_scale: torch.Tensor | None  # float32 [N, H/128] for fp8, else None
    y: torch.Tensor | None        # bf16 [N*k, H]; None for identity experts


def _stream_seed(seed: int, stream: int) -> int:
    """Independent 63-bit seed for one named draw of a workload seed."""
    return int(np.random.SeedSequence([seed, stream]).generate_state(1, np.uint64)[0] >> 1)


def _zipf_log_p(E: int) -> np.ndarray:
    perm = np.random.Generator(np.random.PCG64(0)).permutation(E)
    p = (perm + 1.0) ** (-ZIPF_S)
    p /= p.sum()
    return np.log(p)


def _logits(cfg: Config, seed: int, alpha: float | None) -> np.ndarray:
    rng = np.random.Generator(np.random.PCG64(_stream_seed(seed, 0)))
    z = rng.standard_normal((cfg.N, cfg.E))
    if cfg.routing == "zipf":
        a = ZIPF_ALPHA if alpha is None else alpha
        z = z + a * _zipf_log_p(cfg.E)[None, :]
    elif cfg.routing != "uniform":
        raise ValueError(f"unknown routing {cfg.routing!r}")
    return z


def rank_load_ratio(topk_idx: np.ndarray, E: int, R: int) -> float:
    """max over ranks of routed entries / mean routed entries per rank (skew calibration)."""
    per_rank = np.bincount((topk_idx // (E // R)).ravel(), minlength=R)
    return float(per_rank.max() / (topk_idx.size / R))


def find_zipf_alpha(cfg: Config, seed: int = 0, target: float = SKEW_TARGET,
                    iters: int = 24) -> float:
    """Bisection on alpha so that the busiest rank gets ``target`` x the mean load."""
    lo, hi = 0.0, 8.0
    for _ in range(iters):
        mid = 0.5 * (lo + hi)
        z = _logits(cfg, seed, mid)
        idx = np.argpartition(-z, cfg.k - 1, axis=1)[:, :cfg.k]
        if rank_load_ratio(idx, cfg.E, cfg.R) < target:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


def make_routing(cfg: Config, seed: int, alpha: float | None = None):
    """Top-k expert ids (int32 [N,k], descending logit) and float32 weights [N,k]."""
    z = _logits(cfg, seed, alpha)
    order = np.argsort(-z, axis=1, kind="stable")[:, :cfg.k]
    sel = np.take_along_axis(z, order, axis=1)
    if cfg.weights == "softmax":
        ex = np.exp(sel - sel.max(axis=1, keepdims=True))
        w = ex / ex.sum(axis=1, keepdims=True)
    elif cfg.weights == "sigmoid":
        s = 1.0 / (1.0 + np.exp(-sel))
        w = s / s.sum(axis=1, keepdims=True)
    else:
        raise ValueError(f"unknown weights {cfg.weights!r}")
    return np.ascontiguousarray(order.astype(np.int32)), np.ascontiguousarray(w.astype(np.float32))


def _randn_bf16(rows: int, cols: int, seed: int, device) -> torch.Tensor:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    out = torch.empty((rows, cols), dtype=torch.bfloat16, device=device)
    step = max(1, (1 << 26) // max(cols, 1))
    for r0 in range(0, rows, step):
        r1 = min(rows, r0 + step)
        out[r0:r1] = torch.randn((r1 - r0, cols), generator=g, dtype=torch.float32,
                                 device=device).to(torch.bfloat16)
    return out


def make_payload_x(cfg: Config, seed: int, device="cpu"):
    """(x, x_scale): bf16 [N,H] and None, or fp8 e4m3 bytes uint8 [N,H] and fp32 [N,H/128]."""
    s = _stream_seed(seed, 1)
    if cfg.payload == "bf16":
        return _randn_bf16(cfg.N, cfg.H, s, device), None
    if cfg.payload != "fp8":
        raise ValueError(f"unknown payload {cfg.payload!r}")
    if cfg.H % SCALE_COLS:
        raise ValueError("fp8 payload needs H % 128 == 0")
    g = torch.Generator(device=device)
    g.manual_seed(s)
    nb = cfg.H // SCALE_COLS
    q = torch.empty((cfg.N, cfg.H), dtype=torch.uint8, device=device)
    scale = torch.empty((cfg.N, nb), dtype=torch.float32, device=device)
    step = max(1, (1 << 24) // cfg.H)
    for r0 in range(0, cfg.N, step):
        r1 = min(cfg.N, r0 + step)
        xf = torch.randn((r1 - r0, nb, SCALE_COLS), generator=g, dtype=torch.float32, device=device)
        amax = xf.abs().amax(dim=-1).clamp_min(1e-30)
        sc = amax / FP8_MAX
        q8 = (xf / sc[..., None]).to(torch.float8_e4m3fn)
        q[r0:r1] = q8.reshape(r1 - r0, cfg.H).view(torch.uint8)
        scale[r0:r1] = sc
    return q, scale


def make_payload_y(cfg: Config, seed: int, device="cpu"):
    """Expert outputs: bf16 [N*k, H] ~ N(0,1), or None for identity experts."""
    if cfg.y == "identity":
        return None
    return _randn_bf16(cfg.N * cfg.k, cfg.H, _stream_seed(seed, 2), device)


def make_expert_outputs(rows: int, H: int, seed: int, device="cpu") -> torch.Tensor:
    """bf16 [rows, H] ~ N(0,1): expert outputs for a receive layout of `rows` rows."""
    return _randn_bf16(rows, H, _stream_seed(seed, 2), device)


def drop_entries(topk_idx: np.ndarray, frac: float, seed: int) -> np.ndarray:
    """Mark a seeded fraction of the routing entries as dropped (id -1)."""
    out = topk_idx.copy()
    rng = np.random.Generator(np.random.PCG64(_stream_seed(seed, 3)))
    out[rng.random(out.shape) < frac] = -1
    return out


def make_workload(cfg: Config, seed: int = 0, device="cpu", with_y: bool = True) -> Workload:
    idx, w = make_routing(cfg, seed)
    x, xs = make_payload_x(cfg, seed, device)
    y = make_payload_y(cfg, seed, device) if with_y else None
    return Workload(cfg, seed, idx, w, x, xs, y)


def distinct_rank_expectation(E: int, k: int, R: int) -> float:
    """E[number of distinct ranks a token touches] for k distinct uniform experts.

    A rank holding E/R experts is missed with probability C(E - E/R, k) / C(E, k).
    """
    from math import comb
    return R * (1.0 - comb(E - E // R, k) / comb(E, k))
