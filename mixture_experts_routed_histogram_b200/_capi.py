"""ctypes binding of libmoe.so.  Argument marshalling only: every step of the forward
pass runs in the library's CUDA kernels.  Functions keep the C names; tensors are torch
CUDA tensors (their data pointers are passed), `stream` defaults to torch's current
stream.  A non-OK status raises MoeError.  The library must be built
(``python -m mixture_experts_routed_histogram_b200.build``); there is no fallback."""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoe.so")
_lib = None
_lock = threading.Lock()

MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_UNSUPPORTED_SHAPE = 2
MOE_ERR_MISALIGNED = 3
MOE_ERR_WORKSPACE_TOO_SMALL = 4
MOE_ERR_CUDA = 5
MOE_ERR_DEVICE_TIMEOUT = 6
MOE_ERR_DEVICE_BAD_INDEX = 7

MOE_SCORE_SOFTMAX = 0
MOE_SCORE_SIGMOID = 1
MOE_DTYPE_BF16 = 0
MOE_DTYPE_FP8_MXFP4 = 1
MOE_ACT_SWIGLU = 0
MOE_ACT_RELU2 = 1

# Every function include/moe.h declares.
EXPORTS = ("moe_workspace_size", "moe_workspace_init", "moe_route", "moe_permute",
           "moe_quantize_x", "moe_quantize_weights_mxfp4", "moe_grouped_gemm1_swiglu",
           "moe_grouped_gemm2", "moe_combine", "moe_forward", "moe_get_device_status",
           "moe_status_string", "moe_debug_set_wait_limit_ns", "moe_debug_inject_stall",
           "moe_last_launch_count", "moe_permute_noalloc", "moe_debug_time_stages",
           "moe_debug_stage_times", "moe_workspace_region")

# moe_ws_region_t
MOE_WS_IDS, MOE_WS_W, MOE_WS_COUNTS, MOE_WS_OFFSETS, MOE_WS_ROW2ASSIGN, MOE_WS_ASSIGN2ROW = range(6)


class MoeShape(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("H", ctypes.c_int32), ("I", ctypes.c_int32),
                ("E", ctypes.c_int32), ("k", ctypes.c_int32), ("score", ctypes.c_int32),
                ("renormalize", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("activation", ctypes.c_int32), ("n_shared", ctypes.c_int32)]

    @classmethod
    def of(cls, T, H, I, E, k, score="softmax", renorm=True, dtype="bf16",
           act="swiglu", n_shared=0) -> "MoeShape":
        return cls(int(T), int(H), int(I), int(E), int(k),
                   MOE_SCORE_SOFTMAX if score == "softmax" else MOE_SCORE_SIGMOID,
                   int(bool(renorm)), MOE_DTYPE_BF16 if dtype == "bf16" else MOE_DTYPE_FP8_MXFP4,
                   MOE_ACT_SWIGLU if act == "swiglu" else MOE_ACT_RELU2, int(n_shared))

    @classmethod
    def from_workload(cls, wl) -> "MoeShape":
        return cls.of(wl.T, wl.H, wl.I, wl.E, wl.k, wl.score, wl.renorm, wl.dtype, wl.act,
                      wl.n_shared)


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


def lib_path() -> str:
    return _LIB_PATH


def load():
    """Load libmoe.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(_LIB_PATH):
                raise RuntimeError(f"{_LIB_PATH} is missing: build it with "
                                   "`python -m mixture_experts_routed_histogram_b200.build`")
            L = ctypes.CDLL(_LIB_PATH)
            P, S, vp = ctypes.POINTER, ctypes.POINTER(MoeShape), ctypes.c_void_p
            st, sz = ctypes.c_int, ctypes.c_size_t
            L.moe_workspace_size.argtypes = [S]; L.moe_workspace_size.restype = sz
            L.moe_workspace_init.argtypes = [vp, sz, vp]; L.moe_workspace_init.restype = st
            L.moe_workspace_region.argtypes = [S, ctypes.c_int32, P(sz), P(sz)]
            L.moe_workspace_region.restype = st
            L.moe_route.argtypes = [S, vp, vp, vp, vp]; L.moe_route.restype = st
            L.moe_permute.argtypes = [S, vp, vp, vp, vp, vp, vp, sz, vp]; L.moe_permute.restype = st
            L.moe_permute_noalloc.argtypes = [S, vp, vp, vp, vp, vp, vp]
            L.moe_permute_noalloc.restype = st
            L.moe_quantize_x.argtypes = [S, vp, vp, vp, vp]; L.moe_quantize_x.restype = st
            L.moe_quantize_weights_mxfp4.argtypes = [ctypes.c_int64, ctypes.c_int32, vp, vp, vp, vp]
            L.moe_quantize_weights_mxfp4.restype = st
            L.moe_grouped_gemm1_swiglu.argtypes = [S, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
            L.moe_grouped_gemm1_swiglu.restype = st
            L.moe_grouped_gemm2.argtypes = [S, vp, vp, vp, vp, vp, vp, vp, sz, vp]
            L.moe_grouped_gemm2.restype = st
            L.moe_combine.argtypes = [S, vp, vp, vp, vp, vp]; L.moe_combine.restype = st
            L.moe_forward.argtypes = [S, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
            L.moe_forward.restype = st
            L.moe_get_device_status.argtypes = [vp, vp]; L.moe_get_device_status.restype = st
            L.moe_status_string.argtypes = [st]; L.moe_status_string.restype = ctypes.c_char_p
            L.moe_debug_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
            L.moe_debug_set_wait_limit_ns.restype = None
            L.moe_debug_inject_stall.argtypes = [ctypes.c_int]; L.moe_debug_inject_stall.restype = None
            L.moe_last_launch_count.argtypes = []; L.moe_last_launch_count.restype = ctypes.c_int
            L.moe_debug_time_stages.argtypes = [ctypes.c_int]; L.moe_debug_time_stages.restype = None
            L.moe_debug_stage_times.argtypes = [ctypes.POINTER(ctypes.c_char_p),
                                                ctypes.POINTER(ctypes.c_float), ctypes.c_int]
            L.moe_debug_stage_times.restype = ctypes.c_int
            _lib = L
    return _lib


def _p(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    assert t.is_cuda and t.is_contiguous(), "device tensors must be contiguous CUDA tensors"
    return t.data_ptr()


def _s(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(st: int, where: str):
    if st != MOE_OK:
        raise MoeError(st, where)


def status_string(st: int) -> str:
    try:
        return load().moe_status_string(st).decode()
    except Exception:  # library missing
        return f"status {st}"


def _nbytes(t) -> int:
    return t.numel() * t.element_size()


# ---------------------------------------------------------------- entry points

def moe_workspace_size(shape: MoeShape) -> int:
    return int(load().moe_workspace_size(ctypes.byref(shape)))


def moe_workspace_init(ws, stream=None):
    _check(load().moe_workspace_init(_p(ws), _nbytes(ws), _s(stream)), "moe_workspace_init")


def moe_workspace_region(shape: MoeShape, region: int):
    """(byte offset, bytes) of one routing-metadata region of the forward's workspace."""
    off, n = ctypes.c_size_t(), ctypes.c_size_t()
    _check(load().moe_workspace_region(ctypes.byref(shape), int(region), ctypes.byref(off),
                                       ctypes.byref(n)), "moe_workspace_region")
    return int(off.value), int(n.value)


def moe_route(shape, logits, ids, w, stream=None):
    _check(load().moe_route(ctypes.byref(shape), _p(logits), _p(ids), _p(w), _s(stream)),
           "moe_route")


def moe_permute(shape, ids, counts, offsets, row2assign, assign2row, ws, stream=None):
    _check(load().moe_permute(ctypes.byref(shape), _p(ids), _p(counts), _p(offsets),
                              _p(row2assign), _p(assign2row), _p(ws), _nbytes(ws), _s(stream)),
           "moe_permute")


def moe_permute_noalloc(shape, ids, counts, offsets, row2assign, assign2row, stream=None):
    """moe_permute without a workspace (its scratch is a static device array)."""
    _check(load().moe_permute_noalloc(ctypes.byref(shape), _p(ids), _p(counts), _p(offsets),
                                      _p(row2assign), _p(assign2row), _s(stream)),
           "moe_permute_noalloc")


def moe_quantize_x(shape, x, xq, sx, stream=None):
    _check(load().moe_quantize_x(ctypes.byref(shape), _p(x), _p(xq), _p(sx), _s(stream)),
           "moe_quantize_x")


def moe_quantize_weights_mxfp4(w, packed, sf, stream=None):
    K = w.shape[-1]
    rows = w.numel() // K
    _check(load().moe_quantize_weights_mxfp4(rows, K, _p(w), _p(packed), _p(sf), _s(stream)),
           "moe_quantize_weights_mxfp4")


def moe_grouped_gemm1_swiglu(shape, a, sa, row2assign, offsets, w13, w13_sf, act, act_sf, ws,
                             stream=None):
    _check(load().moe_grouped_gemm1_swiglu(ctypes.byref(shape), _p(a), _p(sa), _p(row2assign),
                                           _p(offsets), _p(w13), _p(w13_sf), _p(act), _p(act_sf),
                                           _p(ws), _nbytes(ws), _s(stream)),
           "moe_grouped_gemm1_swiglu")


def moe_grouped_gemm2(shape, act, act_sf, offsets, w2, w2_sf, y, ws, stream=None):
    _check(load().moe_grouped_gemm2(ctypes.byref(shape), _p(act), _p(act_sf), _p(offsets),
                                    _p(w2), _p(w2_sf), _p(y), _p(ws), _nbytes(ws), _s(stream)),
           "moe_grouped_gemm2")


def moe_combine(shape, y, w, assign2row, out, stream=None):
    _check(load().moe_combine(ctypes.byref(shape), _p(y), _p(w), _p(assign2row), _p(out),
                              _s(stream)), "moe_combine")


def moe_forward(shape, x, logits, w13, w13_sf, w2, w2_sf, out, ids_out, ws, stream=None):
    _check(load().moe_forward(ctypes.byref(shape), _p(x), _p(logits), _p(w13), _p(w13_sf),
                              _p(w2), _p(w2_sf), _p(out), _p(ids_out), _p(ws), _nbytes(ws),
                              _s(stream)), "moe_forward")


def moe_get_device_status(ws, stream=None) -> int:
    return int(load().moe_get_device_status(_p(ws), _s(stream)))


def moe_status_string(st: int) -> str:
    return status_string(st)


def moe_last_launch_count() -> int:
    return int(load().moe_last_launch_count())


def moe_debug_set_wait_limit_ns(ns: int):
    load().moe_debug_set_wait_limit_ns(int(ns))


def moe_debug_inject_stall(on: bool):
    load().moe_debug_inject_stall(int(bool(on)))


def moe_debug_time_stages(on: bool):
    load().moe_debug_time_stages(int(bool(on)))


def moe_debug_stage_times(max_stages: int = 8):
    """[(stage name, ms)] of the last moe_forward recorded on this thread."""
    names = (ctypes.c_char_p * max_stages)()
    ms = (ctypes.c_float * max_stages)()
    n = load().moe_debug_stage_times(names, ms, max_stages)
    if n < 0:
        raise MoeError(MOE_ERR_CUDA, "moe_debug_stage_times")
    return [(names[i].decode(), float(ms[i])) for i in range(min(n, max_stages))]
