"""MoE token shuffle on B200: thin Python binding over libmoeshuffle.so.

Every step (plan, dispatch, combine) runs in the library's CUDA kernels; this module
only checks tensor properties, passes pointers and the current CUDA stream through the
C ABI declared in include/moe_shuffle.h, and allocates outputs with torch when the caller
does not pass them.  There is no CPU fallback: without the built library every call
raises ImportError (the package itself imports, so that its build module can run).

    plan = moe_plan(topk_idx, topk_w, E, R)          # int32 [N,k], fp32 [N,k] on cuda
    recv = moe_dispatch(x, plan)                     # bf16 [N,H] -> [N*k, H]
    out = moe_combine(y, plan)                       # bf16 [N*k,H] -> [N, H]
"""

from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "MoeError", "Plan", "moe_plan", "moe_plan_create", "moe_dispatch", "moe_combine",
    "moe_dispatch_combine", "moe_wait_selftest",
    "moe_tune", "lib_path", "version", "ERR_ID_RANGE", "ERR_ID_DUP", "ERR_BOUNDS",
    "ERR_TIMEOUT", "KNOBS",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libmoeshuffle.so")

MOE_OK, MOE_EINVAL, MOE_ECUDA, MOE_ENOMEM = 0, 1, 2, 3
MOE_BF16, MOE_FP8E4M3 = 0, 1
ERR_ID_RANGE, ERR_ID_DUP, ERR_BOUNDS, ERR_TIMEOUT = 1, 2, 4, 8
KNOBS = {
    "dispatch_stages": 0, "dispatch_lag": 1, "dispatch_ctas_per_sm": 2,
    "dispatch_warps_per_cta": 3, "combine_ctas_per_sm": 5,
    "combine_stages": 6, "combine_smem_kb": 8,
    "dispatch_units_per_warp": 9, "combine_tokens_per_cta": 10, "plan_engine": 11,
    "fused_ctas_per_sm": 12, "fused_dispatch_share": 13, "fused_dispatch_run": 14,
    "fused_combine_run": 15, "fused_smem_kb": 16, "fused_min_kb": 17, "combine_max_cw": 18,
    "plan_cluster": 19, "pdl": 20, "plan_match": 21, "dispatch_split_units": 22,
    "combine_split": 23,
}
PLAN_KINDS = {0: "one_tile", 1: "groups", 2: "cooperative", 3: "three"}

_i32 = ctypes.c_int32
_vp = ctypes.c_void_p


class _PlanView(ctypes.Structure):
    _fields_ = [
        ("N", _i32), ("k", _i32), ("E", _i32), ("R", _i32), ("experts_per_rank", _i32),
        ("capacity_tokens", _i32), ("cnt", _vp), ("expert_off", _vp), ("rcnt", _vp),
        ("rank_off", _vp), ("rtok_off", _vp), ("slot", _vp), ("src_tok", _vp), ("src_j", _vp),
        ("rtok", _vp), ("fanout", _vp), ("err", _vp), ("topk_w", _vp), ("plan_kernels", _i32),
        ("align", _i32), ("recv_rows", _i32), ("plan_kind", _i32), ("dedup_lists", _i32),
    ]


def _load():
    if not os.path.exists(_LIB_PATH):
        raise ImportError(
            f"{_LIB_PATH} is missing: build it with `python -m moe_expert_shuffling_b200.build` "
            "(there is no fallback implementation)")
    lib = ctypes.CDLL(_LIB_PATH)
    st = ctypes.c_int
    lib.moe_plan_create.restype = st
    lib.moe_plan_create.argtypes = [_i32, _i32, _i32, _i32, ctypes.POINTER(_vp)]
    lib.moe_plan_create_aligned.restype = st
    lib.moe_plan_create_aligned.argtypes = [_i32, _i32, _i32, _i32, _i32, ctypes.POINTER(_vp)]
    lib.moe_plan_create_ex.restype = st
    lib.moe_plan_create_ex.argtypes = [_i32, _i32, _i32, _i32, _i32, ctypes.c_uint32,
                                       ctypes.POINTER(_vp)]
    lib.moe_plan.restype = st
    lib.moe_plan.argtypes = [_vp, _vp, _i32, _i32, _i32, _i32, _vp, ctypes.POINTER(_vp)]
    lib.moe_dispatch.restype = st
    lib.moe_dispatch.argtypes = [_vp, ctypes.c_int, _vp, _i32, _vp, _vp, _vp, _vp]
    lib.moe_combine.restype = st
    lib.moe_combine.argtypes = [_vp, _i32, _vp, _vp, _vp]
    lib.moe_combine_ranked.restype = st
    lib.moe_combine_ranked.argtypes = [_vp, _i32, _vp, _vp, _vp]
    lib.moe_dispatch_combine.restype = st
    lib.moe_dispatch_combine.argtypes = [_vp, ctypes.c_int, _vp, _i32, _vp, _vp, _vp, _vp, _i32,
                                         _vp, _vp, _i32, _vp]
    lib.moe_plan_query.restype = st
    lib.moe_plan_query.argtypes = [_vp, ctypes.POINTER(_PlanView)]
    lib.moe_plan_check.restype = st
    lib.moe_plan_check.argtypes = [_vp, _vp, ctypes.POINTER(ctypes.c_uint32)]
    lib.moe_plan_destroy.restype = st
    lib.moe_plan_destroy.argtypes = [_vp]
    lib.moe_last_error.restype = ctypes.c_char_p
    lib.moe_last_error.argtypes = []
    lib.moe_version.restype = ctypes.c_char_p
    lib.moe_version.argtypes = []
    lib.moe_tune.restype = st
    lib.moe_tune.argtypes = [ctypes.c_int, _i32]
    lib.moe_wait_selftest.restype = st
    lib.moe_wait_selftest.argtypes = [_i32, _vp, ctypes.POINTER(ctypes.c_uint32)]
    return lib


class _Library:
    """The library, loaded on first use (so that the package, and its build module, import
    before the library is built or while it is being rebuilt).  Without the built library
    every call fails loudly: there is no fallback implementation."""

    def __init__(self):
        self._handle = None

    def __getattr__(self, name):
        if self._handle is None:
            if not os.path.exists(_LIB_PATH):
                raise ImportError(
                    f"{_LIB_PATH} is missing: build it with "
                    "`python -m moe_expert_shuffling_b200.build` (there is no fallback "
                    "implementation)")
            self._handle = _load()
        return getattr(self._handle, name)


_lib = _Library()


class MoeError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"[status {status}] {message}")
        self.status = status


def _check(status: int) -> None:
    if status != MOE_OK:
        raise MoeError(status, _lib.moe_last_error().decode())


def lib_path() -> str:
    return _LIB_PATH


def version() -> str:
    return _lib.moe_version().decode()


def moe_tune(knob: str, value: int) -> None:
    """Override a launch parameter (speed only, never results); 0 restores the default."""
    _check(_lib.moe_tune(KNOBS[knob], int(value)))


def _stream_ptr(stream) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _need_cuda(t: torch.Tensor, name: str, dtypes, ndim: int | None = None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor (got {t.device})")
    if t.dtype not in dtypes:
        raise TypeError(f"{name} must have dtype in {dtypes} (got {t.dtype})")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims (got {t.dim()})")


class _DeviceArray:
    """Zero-copy export of a plan array to torch (keeps the plan alive)."""

    def __init__(self, ptr: int, n: int, typestr: str, owner):
        self.__cuda_array_interface__ = {
            "shape": (n,), "typestr": typestr, "data": (ptr, False), "version": 3,
            "strides": None, "stream": None,
        }
        self._owner = owner


class Plan:
    """Owner of a moe_plan_t.  Holds references to the routing tensors it was built from."""

    def __init__(self, handle: int):
        self._h = _vp(handle)
        self._refs = ()
        self._meta = None  # (N, k, E, R, rows) of the last plan, cached for the hot calls

    def _cached(self):
        if self._meta is None:
            v = self._view()
            self._meta = (v.N, v.k, v.E, v.R, v.recv_rows)
        return self._meta

    @property
    def handle(self) -> int:
        return self._h.value or 0

    def _view(self) -> _PlanView:
        v = _PlanView()
        _check(_lib.moe_plan_query(self._h, ctypes.byref(v)))
        return v

    @property
    def shape(self) -> tuple[int, int, int, int]:
        return self._cached()[:4]

    @property
    def capacity(self) -> int:
        return self._view().capacity_tokens

    @property
    def rows(self) -> int:
        """Rows a receive buffer needs for the last plan: N*k + E*(align - 1)."""
        return self._cached()[4]

    @property
    def align(self) -> int:
        return self._view().align

    @property
    def plan_kernels(self) -> int:
        """Kernels the last moe_plan call enqueued (1, or 3)."""
        return self._view().plan_kernels

    @property
    def plan_kind(self) -> str:
        """Planner kernel of the last moe_plan call: one_tile, groups, cooperative or three."""
        return PLAN_KINDS[self._view().plan_kind]

    @property
    def dedup_lists(self) -> bool:
        """Whether moe_plan writes the per-rank lists rtok / fanout."""
        return bool(self._view().dedup_lists)

    def arrays(self) -> dict[str, torch.Tensor]:
        """Zero-copy int32 views of the plan's device arrays (fanout/err as bit patterns)."""
        v = self._view()
        N, k, E, R = v.N, v.k, v.E, v.R
        dev = torch.device("cuda", torch.cuda.current_device())

        def arr(ptr, n):
            if n == 0:
                return torch.empty(0, dtype=torch.int32, device=dev)
            return torch.as_tensor(_DeviceArray(ptr, n, "<i4", self), device=dev)

        rtok_off = arr(v.rtok_off, R + 1)
        n_dedup = int(rtok_off[-1].item())
        return {
            "cnt": arr(v.cnt, E), "expert_off": arr(v.expert_off, E + 1),
            "rcnt": arr(v.rcnt, R), "rank_off": arr(v.rank_off, R + 1),
            "rtok_off": rtok_off, "slot": arr(v.slot, N * k).view(N, k) if N else
            torch.empty((0, k), dtype=torch.int32, device=dev),
            "src_tok": arr(v.src_tok, v.recv_rows), "src_j": arr(v.src_j, v.recv_rows),
            "rtok": arr(v.rtok, n_dedup), "fanout": arr(v.fanout, n_dedup),
            "err": arr(v.err, 1),
        }

    def check(self, stream=None) -> int:
        """Synchronise `stream` and return the plan's MOE_ERR_* bits (0 = all good)."""
        flags = ctypes.c_uint32(0)
        _check(_lib.moe_plan_check(self._h, _vp(_stream_ptr(stream)), ctypes.byref(flags)))
        return int(flags.value)

    def close(self) -> None:
        if self._h and self._h.value:
            _lib.moe_plan_destroy(self._h)
            self._h = _vp(0)
        self._refs = ()

    def __del__(self):  # pragma: no cover - interpreter shutdown order varies
        try:
            self.close()
        except Exception:
            pass


PLAN_NO_DEDUP_LISTS = 1


def moe_plan_create(max_tokens: int, k: int, E: int, R: int, align: int = 1,
                    dedup_lists: bool = True) -> Plan:
    """Allocate a reusable plan; with align > 1 expert segments start on multiples of it;
    with dedup_lists=False moe_plan skips the per-rank lists rtok / fanout."""
    h = _vp(0)
    flags = 0 if dedup_lists else PLAN_NO_DEDUP_LISTS
    _check(_lib.moe_plan_create_ex(int(max_tokens), int(k), int(E), int(R), int(align), flags,
                                   ctypes.byref(h)))
    return Plan(h.value)


def moe_plan(topk_idx: torch.Tensor, topk_w: torch.Tensor, E: int, R: int,
             plan: Plan | None = None, stream=None) -> Plan:
    """Build the segment plan of one routing on the current stream (see moe_plan in the C ABI)."""
    _need_cuda(topk_idx, "topk_idx", (torch.int32,), 2)
    _need_cuda(topk_w, "topk_w", (torch.float32,), 2)
    if topk_w.shape != topk_idx.shape:
        raise ValueError("topk_w must have the shape of topk_idx")
    N, k = topk_idx.shape
    h = _vp(plan.handle if plan is not None else 0)
    _check(_lib.moe_plan(_vp(topk_idx.data_ptr()), _vp(topk_w.data_ptr()), N, k, int(E), int(R),
                         _vp(_stream_ptr(stream)), ctypes.byref(h)))
    if plan is None:
        plan = Plan(h.value)
    plan._refs = (topk_idx, topk_w)
    if plan._meta is None or plan._meta[0] != N:
        plan._meta = None
    return plan


def moe_dispatch(x: torch.Tensor, plan: Plan, recv: torch.Tensor | None = None,
                 x_scale: torch.Tensor | None = None, recv_scale: torch.Tensor | None = None,
                 stream=None):
    """recv[slot[t,j]] = x[t].  bf16 returns recv; fp8 (uint8 / float8_e4m3fn) returns (recv, recv_scale)."""
    _need_cuda(x, "x", (torch.bfloat16, torch.uint8, torch.float8_e4m3fn), 2)
    N, H = x.shape
    pN, k, _, _ = plan.shape
    if N != pN:
        raise ValueError(f"x has {N} rows but the plan has {pN} tokens")
    fp8 = x.dtype != torch.bfloat16
    rows = plan.rows
    if recv is None:
        recv = torch.empty((rows, H), dtype=x.dtype, device=x.device)
    _need_cuda(recv, "recv", (x.dtype,), 2)
    if tuple(recv.shape) != (rows, H):
        raise ValueError(f"recv must have shape {(rows, H)}")
    xs_ptr = rs_ptr = 0
    if fp8:
        if x_scale is None:
            raise ValueError("fp8 dispatch needs x_scale [N, H/128]")
        _need_cuda(x_scale, "x_scale", (torch.float32,), 2)
        if tuple(x_scale.shape) != (N, H // 128):
            raise ValueError(f"x_scale must have shape {(N, H // 128)}")
        if recv_scale is None:
            recv_scale = torch.empty((rows, H // 128), dtype=torch.float32, device=x.device)
        _need_cuda(recv_scale, "recv_scale", (torch.float32,), 2)
        if tuple(recv_scale.shape) != (rows, H // 128):
            raise ValueError(f"recv_scale must have shape {(rows, H // 128)}")
        xs_ptr, rs_ptr = x_scale.data_ptr(), recv_scale.data_ptr()
    _check(_lib.moe_dispatch(_vp(x.data_ptr()), MOE_FP8E4M3 if fp8 else MOE_BF16, _vp(xs_ptr),
                             H, plan._h, _vp(recv.data_ptr()), _vp(rs_ptr),
                             _vp(_stream_ptr(stream))))
    return (recv, recv_scale) if fp8 else recv


def moe_combine(y: torch.Tensor, plan: Plan, out: torch.Tensor | None = None, stream=None,
                ranked: bool = False):
    """out[t] = bf16(sum_j w[t,j] * y[slot[t,j]]) with an fp32 fma chain in column order;
    with ranked=True the sum is grouped by rank first (moe_combine_ranked)."""
    _need_cuda(y, "y", (torch.bfloat16,), 2)
    N, k, _, _ = plan.shape
    rows, H = y.shape
    if rows != plan.rows:
        raise ValueError(f"y must have {plan.rows} rows (got {rows})")
    if out is None:
        out = torch.empty((N, H), dtype=torch.bfloat16, device=y.device)
    _need_cuda(out, "out", (torch.bfloat16,), 2)
    if tuple(out.shape) != (N, H):
        raise ValueError(f"out must have shape {(N, H)}")
    fn = _lib.moe_combine_ranked if ranked else _lib.moe_combine
    _check(fn(_vp(y.data_ptr()), H, plan._h, _vp(out.data_ptr()), _vp(_stream_ptr(stream))))
    return out


def moe_dispatch_combine(x: torch.Tensor, dispatch_plan: Plan, recv: torch.Tensor,
                         y: torch.Tensor, combine_plan: Plan, out: torch.Tensor | None = None,
                         x_scale: torch.Tensor | None = None,
                         recv_scale: torch.Tensor | None = None, ranked: bool = False,
                         stream=None):
    """moe_dispatch(x, dispatch_plan, recv) and moe_combine(y, combine_plan, out) in one
    launch.  Pass y=recv (with one plan) to combine the rows this call dispatches.
    Returns out (and recv_scale for fp8 rows)."""
    _need_cuda(x, "x", (torch.bfloat16, torch.uint8, torch.float8_e4m3fn), 2)
    _need_cuda(y, "y", (torch.bfloat16,), 2)
    N, H = x.shape
    if N != dispatch_plan.shape[0]:
        raise ValueError(f"x has {N} rows but the dispatch plan has {dispatch_plan.shape[0]} tokens")
    fp8 = x.dtype != torch.bfloat16
    _need_cuda(recv, "recv", (x.dtype,), 2)
    if tuple(recv.shape) != (dispatch_plan.rows, H):
        raise ValueError(f"recv must have shape {(dispatch_plan.rows, H)}")
    xs_ptr = rs_ptr = 0
    if fp8:
        if x_scale is None:
            raise ValueError("fp8 dispatch needs x_scale [N, H/128]")
        _need_cuda(x_scale, "x_scale", (torch.float32,), 2)
        if tuple(x_scale.shape) != (N, H // 128):
            raise ValueError(f"x_scale must have shape {(N, H // 128)}")
        if recv_scale is None:
            recv_scale = torch.empty((dispatch_plan.rows, H // 128), dtype=torch.float32,
                                     device=x.device)
        _need_cuda(recv_scale, "recv_scale", (torch.float32,), 2)
        if tuple(recv_scale.shape) != (dispatch_plan.rows, H // 128):
            raise ValueError(f"recv_scale must have shape {(dispatch_plan.rows, H // 128)}")
        xs_ptr, rs_ptr = x_scale.data_ptr(), recv_scale.data_ptr()
    Nc = combine_plan.shape[0]
    rows, Hy = y.shape
    if rows != combine_plan.rows:
        raise ValueError(f"y must have {combine_plan.rows} rows (got {rows})")
    if out is None:
        out = torch.empty((Nc, Hy), dtype=torch.bfloat16, device=y.device)
    _need_cuda(out, "out", (torch.bfloat16,), 2)
    if tuple(out.shape) != (Nc, Hy):
        raise ValueError(f"out must have shape {(Nc, Hy)}")
    _check(_lib.moe_dispatch_combine(
        _vp(x.data_ptr()), MOE_FP8E4M3 if fp8 else MOE_BF16, _vp(xs_ptr), H, dispatch_plan._h,
        _vp(recv.data_ptr()), _vp(rs_ptr), _vp(y.data_ptr()), Hy, combine_plan._h,
        _vp(out.data_ptr()), 1 if ranked else 0, _vp(_stream_ptr(stream))))
    return (out, recv_scale) if fp8 else out


def moe_wait_selftest(which: int, stream=None) -> int:
    """Run one bounded device wait on something that never completes (0: ready flag,
    1: mbarrier, 2: grid barrier) and return the error word it leaves (ERR_TIMEOUT when the
    wait gave up).  Blocks for about a second."""
    flags = ctypes.c_uint32(0)
    _check(_lib.moe_wait_selftest(which, _vp(_stream_ptr(stream)), ctypes.byref(flags)))
    return flags.value
