"""Python binding of libmoe_b200.so, the C-ABI int4 expert-grouped MoE layer.

Argument marshalling only: every step of the layer runs in the library's
CUDA kernels.  Tensors are torch tensors (device memory and streams come
from torch); they are passed to the C entry points as raw pointers.  There is
no fallback: importing this package without the built library raises.

Entry points (same names as include/moe.h):
    Plan(shape)                       moe_plan_create / moe_plan_info
    Plan.prepack_weights(...)         moe_prepack_weights
    Plan.route(...)                   moe_route
    Plan.forward(...)                 moe_forward
    Plan.forward_host(...)            moe_forward_host
    Plan.read_status(ws)              moe_read_status
    Plan.dispatch(...)                moe_dispatch         (expert parallelism,
    Plan.experts_forward(...)         moe_experts_forward   see ep.py)
    Plan.combine(...)                 moe_combine
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        "libmoe_b200.so is not built; run `python int4_expert_grouped_b200/build.py` "
        "(needs nvcc with sm_100a support)")

_lib = ctypes.CDLL(LIB_PATH)

MOE_OK = 0
SHAPE_TEST_TIMEOUT = 1  # MOE_SHAPE_TEST_TIMEOUT: test hook of the bounded-wait path
STATUS_NAMES = {
    0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED_SHAPE",
    3: "MOE_ERR_ALIGNMENT", 4: "MOE_ERR_WORKSPACE_TOO_SMALL", 5: "MOE_ERR_CUDA",
    6: "MOE_ERR_DEVICE_TIMEOUT", 7: "MOE_ERR_DEVICE_BOUNDS",
}


class MoeError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__("%s failed: %s (%s)" % (where, STATUS_NAMES.get(code, code),
                                                 _lib.moe_status_str(code).decode()))


class Shape(ctypes.Structure):
    _fields_ = [("T_max", ctypes.c_int32), ("d", ctypes.c_int32), ("E", ctypes.c_int32),
                ("k", ctypes.c_int32), ("f", ctypes.c_int32), ("group", ctypes.c_int32),
                ("flags", ctypes.c_uint32)]


class PlanInfo(ctypes.Structure):
    _fields_ = [("workspace_bytes", ctypes.c_size_t), ("host_workspace_bytes", ctypes.c_size_t),
                ("packed_weight_bytes", ctypes.c_size_t), ("block_t", ctypes.c_int32),
                ("max_blocks", ctypes.c_int32)]


class Projection(ctypes.Structure):
    _fields_ = [("q", ctypes.c_void_p), ("scale", ctypes.c_void_p), ("bias", ctypes.c_void_p)]


class ExpertWeights(ctypes.Structure):
    _fields_ = [("gate", Projection), ("up", Projection), ("down", Projection)]


class StageEvents(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("start", "routed", "gate_up", "down", "end")]


class RouteOut(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "topk_idx", "topk_w", "counts", "offsets", "sorted_assign", "pos",
        "block_offsets", "block_map", "num_blocks")]


_P = ctypes.c_void_p
_lib.moe_abi_version.restype = ctypes.c_int
_lib.moe_status_str.restype = ctypes.c_char_p
_lib.moe_status_str.argtypes = [ctypes.c_int]
_lib.moe_plan_create.argtypes = [ctypes.POINTER(Shape), ctypes.POINTER(_P), ctypes.POINTER(PlanInfo)]
_lib.moe_plan_info.argtypes = [_P, ctypes.POINTER(PlanInfo)]
_lib.moe_plan_destroy.argtypes = [_P]
_lib.moe_plan_destroy.restype = None
_lib.moe_prepack_weights.argtypes = [_P, ctypes.POINTER(ExpertWeights), _P, _P]
_lib.moe_route.argtypes = [_P, ctypes.c_int32, _P, _P, _P, ctypes.POINTER(RouteOut), _P,
                           ctypes.c_size_t, _P]
_lib.moe_forward.argtypes = [_P, ctypes.c_int32, _P, _P, _P, _P, _P, ctypes.POINTER(RouteOut),
                             _P, ctypes.c_size_t, _P]
_lib.moe_forward_timed.argtypes = [_P, ctypes.c_int32, _P, _P, _P, _P, _P,
                                   ctypes.POINTER(RouteOut), _P, ctypes.c_size_t, _P,
                                   ctypes.POINTER(StageEvents)]
_lib.moe_route_noalloc.argtypes = [_P, ctypes.c_int32, _P, _P, _P, ctypes.POINTER(RouteOut), _P]
_lib.moe_forward_host.argtypes = [_P, ctypes.c_int32, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]
_lib.moe_read_status.argtypes = [_P, ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int32),
                                 ctypes.c_int32, _P]
_lib.moe_dispatch.argtypes = [_P, ctypes.c_int32, _P, _P, _P, _P, ctypes.c_size_t, _P]
_lib.moe_experts_forward.argtypes = [_P, ctypes.c_int32, _P, _P, _P, ctypes.c_int32, _P, _P, _P,
                                     ctypes.c_size_t, _P]
_lib.moe_combine.argtypes = [_P, ctypes.c_int32, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]
_lib.moe_forward_path.argtypes = [_P, ctypes.c_int32]
_lib.moe_forward_path.restype = ctypes.c_int
for _fn in ("moe_plan_create", "moe_plan_info", "moe_prepack_weights", "moe_route",
            "moe_forward", "moe_forward_timed", "moe_forward_host", "moe_read_status",
            "moe_route_noalloc", "moe_dispatch", "moe_experts_forward", "moe_combine"):
    getattr(_lib, _fn).restype = ctypes.c_int

EXPORTED = ("moe_abi_version", "moe_status_str", "moe_plan_create", "moe_plan_info",
            "moe_plan_destroy", "moe_prepack_weights", "moe_route", "moe_forward",
            "moe_forward_timed", "moe_forward_host", "moe_read_status", "moe_route_noalloc",
            "moe_forward_path", "moe_dispatch", "moe_experts_forward", "moe_combine")


def abi_version() -> int:
    return _lib.moe_abi_version()


def lib():
    return _lib


def ptr(t) -> int | None:
    """Raw address of a torch tensor / numpy array, an int, or None."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if hasattr(t, "data_ptr"):
        return t.data_ptr()
    if hasattr(t, "ctypes"):
        return t.ctypes.data
    raise TypeError("cannot take the address of %r" % type(t))


def _stream_ptr(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(code: int, where: str):
    if code != MOE_OK:
        raise MoeError(code, where)


class Plan:
    """moe_plan_create for one layer shape (host only, touches no GPU)."""

    def __init__(self, T_max: int, d: int, E: int, k: int, f: int, group: int, flags: int = 0):
        self.shape = Shape(T_max, d, E, k, f, group, flags)
        self._h = _P()
        self.info = PlanInfo()
        _check(_lib.moe_plan_create(ctypes.byref(self.shape), ctypes.byref(self._h),
                                    ctypes.byref(self.info)), "moe_plan_create")

    def __del__(self):
        h = getattr(self, "_h", None)
        if h is not None and h.value:
            _lib.moe_plan_destroy(h)
            self._h = _P()

    @property
    def handle(self):
        return self._h

    def prepack_weights(self, gate, up, down, packed_out, stream=None):
        """gate/up/down: (q, scale, bias) device tensors in the logical layout."""
        w = ExpertWeights(Projection(*[ptr(t) for t in gate]), Projection(*[ptr(t) for t in up]),
                          Projection(*[ptr(t) for t in down]))
        _check(_lib.moe_prepack_weights(self._h, ctypes.byref(w), ptr(packed_out),
                                        _stream_ptr(stream)), "moe_prepack_weights")

    @staticmethod
    def route_out(bufs: dict | None):
        if bufs is None:
            return None
        return RouteOut(*[ptr(bufs[n]) for n, _ in RouteOut._fields_])

    def route(self, T, x, w_r, b_r, out: dict, ws, stream=None):
        ro = self.route_out(out)
        _check(_lib.moe_route(self._h, T, ptr(x), ptr(w_r), ptr(b_r), ctypes.byref(ro), ptr(ws),
                              ws.numel() * ws.element_size(), _stream_ptr(stream)), "moe_route")

    def route_noalloc(self, T, x, w_r, b_r, out: dict, stream=None):
        """moe_route_noalloc: routing with the library's own fixed scratch."""
        ro = self.route_out(out)
        _check(_lib.moe_route_noalloc(self._h, T, ptr(x), ptr(w_r), ptr(b_r), ctypes.byref(ro),
                                      _stream_ptr(stream)), "moe_route_noalloc")

    def forward(self, T, x, w_r, b_r, packed_w, y, ws, route_out: dict | None = None, stream=None,
                events=None):
        """events: None, or five torch.cuda.Event (start, routed, gate_up,
        down, end) recorded between the stages (moe_forward_timed)."""
        ro = self.route_out(route_out)
        ro_p = ctypes.byref(ro) if ro is not None else None
        args = (self._h, T, ptr(x), ptr(w_r), ptr(b_r), ptr(packed_w), ptr(y), ro_p, ptr(ws),
                ws.numel() * ws.element_size(), _stream_ptr(stream))
        if events is None:
            _check(_lib.moe_forward(*args), "moe_forward")
        else:
            ev = StageEvents(*[e.cuda_event if e is not None else None for e in events])
            _check(_lib.moe_forward_timed(*args, ctypes.byref(ev)), "moe_forward_timed")

    def forward_host(self, T, x_host, w_r, b_r, packed_w, y_host, ws, stream=None):
        _check(_lib.moe_forward_host(self._h, T, ptr(x_host), ptr(w_r), ptr(b_r), ptr(packed_w),
                                     ptr(y_host), ptr(ws), ws.numel() * ws.element_size(),
                                     _stream_ptr(stream)), "moe_forward_host")

    def dispatch(self, T, x, sorted_assign, xs, ws, stream=None):
        """moe_dispatch: xs[p] = x[sorted_assign[p] / k]."""
        _check(_lib.moe_dispatch(self._h, T, ptr(x), ptr(sorted_assign), ptr(xs), ptr(ws),
                                 ws.numel() * ws.element_size(), _stream_ptr(stream)), "moe_dispatch")

    def experts_forward(self, rows, xs, block_map, num_blocks, packed_w, o, ws, stream=None):
        """moe_experts_forward over `rows` rows of xs; block_map int32 [n, 3] and
        num_blocks int32 [>= 1] on the device (max_blocks = n)."""
        _check(_lib.moe_experts_forward(self._h, rows, ptr(xs), ptr(block_map), ptr(num_blocks),
                                        int(block_map.shape[0]), ptr(packed_w), ptr(o), ptr(ws),
                                        ws.numel() * ws.element_size(), _stream_ptr(stream)),
               "moe_experts_forward")

    def combine(self, T, o, pos, topk_w, y, ws, stream=None):
        """moe_combine: y[t] = bf16(sum_j topk_w[t, j] o[pos[t k + j]])."""
        _check(_lib.moe_combine(self._h, T, ptr(o), ptr(pos), ptr(topk_w), ptr(y), ptr(ws),
                                ws.numel() * ws.element_size(), _stream_ptr(stream)), "moe_combine")

    def forward_path(self, T: int) -> int:
        """1 if moe_forward runs the small-batch kernels at batch T, 0 for the batched ones."""
        return int(_lib.moe_forward_path(self._h, T))

    def read_status(self, ws, clear: bool = True, stream=None):
        code = ctypes.c_int32()
        detail = ctypes.c_int32()
        _check(_lib.moe_read_status(ptr(ws), ctypes.byref(code), ctypes.byref(detail),
                                    1 if clear else 0, _stream_ptr(stream)), "moe_read_status")
        return code.value, detail.value
