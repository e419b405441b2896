"""CPU oracle for the MoE token shuffle -- TEST INFRASTRUCTURE ONLY.

Plain, slow, single-threaded C loops (oracle.c) behind a numpy interface.  Only the
tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg use it; the
CUDA library neither imports nor links it.  Every function follows the definitions
cited in oracle.c (FUSCO abstract and summary for the segment plan and the fused
dispatch; the DySHARP blog, sections 1-2, for combine and per-rank dedup).
"""

from __future__ import annotations

import ctypes
import os
from contextlib import contextmanager
from dataclasses import dataclass

import numpy as np

from .build import build as _build

_i32p = ctypes.POINTER(ctypes.c_int32)
_u32p = ctypes.POINTER(ctypes.c_uint32)
_u16p = ctypes.POINTER(ctypes.c_uint16)
_u8p = ctypes.POINTER(ctypes.c_uint8)
_f32p = ctypes.POINTER(ctypes.c_float)
_f64p = ctypes.POINTER(ctypes.c_double)
_i64 = ctypes.c_int64
_i32 = ctypes.c_int32


def _bind(path: str):
    lib = ctypes.CDLL(path)
    lib.oracle_plan.restype = ctypes.c_int
    lib.oracle_plan.argtypes = [_i32p, _i64, _i32, _i32, _i32, _i32p, _i32p, _i32p, _i32p,
                                _i32p, _i32p, _i32p, _i32p, _i32p, _u32p, _i64]
    lib.oracle_plan_ex.restype = ctypes.c_int
    lib.oracle_plan_ex.argtypes = [_i32p, _i64, _i32, _i32, _i32, _i32, _i32p, _i32p, _i32p,
                                   _i32p, _i32p, _i32p, _i32p, _i32p, _i32p, _u32p, _i64]
    lib.oracle_validate.restype = ctypes.c_int
    lib.oracle_validate.argtypes = [_i32p, _i64, _i32, _i32]
    lib.oracle_dedup_count.restype = ctypes.c_int64
    lib.oracle_dedup_count.argtypes = [_i32p, _i64, _i32, _i32, _i32]
    lib.oracle_dispatch.restype = None
    lib.oracle_dispatch.argtypes = [_u8p, _u8p, _i32p, _i64, _i32, _i64, _i64, _u8p, _u8p]
    lib.oracle_combine.restype = None
    lib.oracle_combine.argtypes = [_u16p, _i32p, _f32p, _i64, _i32, _i64, _u16p]
    lib.oracle_combine_ranked.restype = None
    lib.oracle_combine_ranked.argtypes = [_u16p, _i32p, _f32p, _i32p, _i64, _i32, _i64, _i32,
                                          _i32, _u16p]
    lib.oracle_combine_f64.restype = None
    lib.oracle_combine_f64.argtypes = [_u16p, _i32p, _f32p, _i64, _i32, _i64, _f64p]
    lib.oracle_f32_to_bf16.restype = None
    lib.oracle_f32_to_bf16.argtypes = [_f32p, _i64, _u16p]
    return lib


_DEFAULT = None


def _lib():
    global _DEFAULT
    if _DEFAULT is None:
        _DEFAULT = _bind(_build())
    return _DEFAULT


@contextmanager
def using_library(path: str):
    """Run the oracle functions on another build of oracle.c for the duration of the block
    (the pin tests use this to check that planted mistakes are caught)."""
    global _DEFAULT
    prev = _lib()
    _DEFAULT = _bind(path)
    try:
        yield
    finally:
        _DEFAULT = prev


def _p(a: np.ndarray, ptype):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ptype)


class OracleError(ValueError):
    pass


@dataclass
class Plan:
    N: int
    k: int
    E: int
    R: int
    cnt: np.ndarray         # int32 [E]
    expert_off: np.ndarray  # int32 [E+1]
    rcnt: np.ndarray        # int32 [R]
    rank_off: np.ndarray    # int32 [R+1]
    rtok_off: np.ndarray    # int32 [R+1]
    slot: np.ndarray        # int32 [N, k] (-1 for a dropped entry)
    src_tok: np.ndarray     # int32 [rows] (-1 for padding and unused rows)
    src_j: np.ndarray       # int32 [rows]
    rtok: np.ndarray        # int32 [sum rcnt]
    fanout: np.ndarray      # uint32 [sum rcnt]
    align: int = 1

    @property
    def rows(self) -> int:
        """Receive rows a buffer must hold: N*k + E*(align - 1)."""
        return self.N * self.k + self.E * (self.align - 1)


def validate(topk_idx: np.ndarray, E: int) -> bool:
    idx = np.ascontiguousarray(topk_idx, dtype=np.int32)
    N, k = idx.shape
    return bool(_lib().oracle_validate(_p(idx, _i32p), N, k, E))


def dedup_count(topk_idx: np.ndarray, E: int, R: int) -> int:
    idx = np.ascontiguousarray(topk_idx, dtype=np.int32)
    N, k = idx.shape
    return int(_lib().oracle_dedup_count(_p(idx, _i32p), N, k, E, R))


def plan(topk_idx: np.ndarray, E: int, R: int, align: int = 1) -> Plan:
    """The segment plan; ids of -1 are dropped entries; segments start on multiples of align."""
    idx = np.ascontiguousarray(topk_idx, dtype=np.int32)
    N, k = idx.shape
    cap = max(1, N * min(k, R))
    rows = N * k + E * (max(align, 1) - 1)
    cnt = np.zeros(E, np.int32)
    expert_off = np.zeros(E + 1, np.int32)
    rcnt = np.zeros(R, np.int32)
    rank_off = np.zeros(R + 1, np.int32)
    rtok_off = np.zeros(R + 1, np.int32)
    slot = np.zeros((N, k), np.int32)
    src_tok = np.zeros(max(1, rows), np.int32)
    src_j = np.zeros(max(1, rows), np.int32)
    rtok = np.zeros(cap, np.int32)
    fanout = np.zeros(cap, np.uint32)
    rc = _lib().oracle_plan_ex(_p(idx, _i32p), N, k, E, R, align, _p(cnt, _i32p),
                               _p(expert_off, _i32p), _p(rcnt, _i32p), _p(rank_off, _i32p),
                               _p(rtok_off, _i32p), _p(slot, _i32p), _p(src_tok, _i32p),
                               _p(src_j, _i32p), _p(rtok, _i32p), _p(fanout, _u32p), cap)
    if rc != 0:
        raise OracleError("invalid routing or shape")
    n = int(rtok_off[R])
    return Plan(N, k, E, R, cnt, expert_off, rcnt, rank_off, rtok_off, slot,
                src_tok[:rows].copy(), src_j[:rows].copy(), rtok[:n].copy(), fanout[:n].copy(),
                align)


def dispatch(x_rows: np.ndarray, slot: np.ndarray, x_scale_rows: np.ndarray | None = None,
             rows: int | None = None):
    """x_rows: uint8 [N, row_bytes]; returns recv uint8 [rows, row_bytes] (and scales), rows
    defaulting to N*k; rows no entry maps to stay zero."""
    x = np.ascontiguousarray(x_rows.view(np.uint8).reshape(x_rows.shape[0], -1))
    sl = np.ascontiguousarray(slot, dtype=np.int32)
    N, k = sl.shape
    rb = x.shape[1]
    nrows = N * k if rows is None else rows
    recv = np.zeros((nrows, rb), np.uint8)
    if x_scale_rows is not None:
        xs = np.ascontiguousarray(x_scale_rows.view(np.uint8).reshape(N, -1))
        sb = xs.shape[1]
        rs = np.zeros((nrows, sb), np.uint8)
        _lib().oracle_dispatch(_p(x, _u8p), _p(xs, _u8p), _p(sl, _i32p), N, k, rb, sb,
                               _p(recv, _u8p), _p(rs, _u8p))
        return recv, rs
    dummy = np.zeros(1, np.uint8)
    _lib().oracle_dispatch(_p(x, _u8p), _p(dummy, _u8p), _p(sl, _i32p), N, k, rb, 0,
                           _p(recv, _u8p), _p(dummy, _u8p))
    return recv


def combine(y_bf16_bits: np.ndarray, slot: np.ndarray, w: np.ndarray) -> np.ndarray:
    """y: uint16 [N*k, H] bf16 bit patterns; returns out uint16 [N, H]."""
    y = np.ascontiguousarray(y_bf16_bits.view(np.uint16))
    sl = np.ascontiguousarray(slot, dtype=np.int32)
    ww = np.ascontiguousarray(w, dtype=np.float32)
    N, k = sl.shape
    H = y.shape[1]
    out = np.zeros((N, H), np.uint16)
    _lib().oracle_combine(_p(y, _u16p), _p(sl, _i32p), _p(ww, _f32p), N, k, H, _p(out, _u16p))
    return out


def combine_ranked(y_bf16_bits: np.ndarray, slot: np.ndarray, w: np.ndarray,
                   topk_idx: np.ndarray, E: int, R: int) -> np.ndarray:
    """Rank-grouped combine: per-rank fp32 fma chains, then fp32 adds across ranks."""
    y = np.ascontiguousarray(y_bf16_bits.view(np.uint16))
    sl = np.ascontiguousarray(slot, dtype=np.int32)
    ww = np.ascontiguousarray(w, dtype=np.float32)
    idx = np.ascontiguousarray(topk_idx, dtype=np.int32)
    N, k = sl.shape
    H = y.shape[1]
    out = np.zeros((N, H), np.uint16)
    _lib().oracle_combine_ranked(_p(y, _u16p), _p(sl, _i32p), _p(ww, _f32p), _p(idx, _i32p), N,
                                 k, H, E, R, _p(out, _u16p))
    return out


def combine_f64(y_bf16_bits: np.ndarray, slot: np.ndarray, w: np.ndarray) -> np.ndarray:
    y = np.ascontiguousarray(y_bf16_bits.view(np.uint16))
    sl = np.ascontiguousarray(slot, dtype=np.int32)
    ww = np.ascontiguousarray(w, dtype=np.float32)
    N, k = sl.shape
    H = y.shape[1]
    out = np.zeros((N, H), np.float64)
    _lib().oracle_combine_f64(_p(y, _u16p), _p(sl, _i32p), _p(ww, _f32p), N, k, H,
                              _p(out, _f64p))
    return out


def f32_to_bf16(a: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(a, dtype=np.float32)
    out = np.zeros(x.shape, np.uint16)
    _lib().oracle_f32_to_bf16(_p(x, _f32p), x.size, _p(out, _u16p))
    return out


def lib_path() -> str:
    return os.path.abspath(_build())
