"""fp64 CPU oracle for the routed-expert MoE MLP forward pass (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
import this package.  The product path (the CUDA library and its Python binding) never
touches it, and it shares no code with them.

The arithmetic lives in ``moe_oracle.c`` (plain C, double precision, OpenMP over tokens);
this module only compiles it on demand and marshals numpy arrays through ctypes.  Each
wrapper names the step of the method it follows; the C file's header gives the passages.

Parity status of every function: pinned by ``tests/test_oracle_pins.py`` (closed forms,
library routines for the number formats, brute force on tiny inputs, invariants and the
block-scaled -> BF16 reduction).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_SO = os.path.join(_HERE, "libmoe_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile moe_oracle.c into libmoe_oracle.so (gcc -O2, OpenMP, no fast-math)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _SO)
    return _SO


def _P(t):
    return ctypes.POINTER(t)


def lib():
    global _lib
    with _lock:
        if _lib is None:
            L = ctypes.CDLL(build())
            i64, i32, f64, u8, u16, f32 = (ctypes.c_int64, ctypes.c_int, ctypes.c_double,
                                           ctypes.c_uint8, ctypes.c_uint16, ctypes.c_float)
            L.orc_bf16_to_f64.argtypes = [u16]; L.orc_bf16_to_f64.restype = f64
            L.orc_f64_to_bf16_rne.argtypes = [f64]; L.orc_f64_to_bf16_rne.restype = u16
            L.orc_e4m3_decode.argtypes = [u8]; L.orc_e4m3_decode.restype = f64
            L.orc_e4m3_encode_rne_satfinite.argtypes = [f64]; L.orc_e4m3_encode_rne_satfinite.restype = u8
            L.orc_e2m1_decode.argtypes = [u8]; L.orc_e2m1_decode.restype = f64
            L.orc_e2m1_encode_rne_satfinite.argtypes = [f64]; L.orc_e2m1_encode_rne_satfinite.restype = u8
            L.orc_ue8m0_decode.argtypes = [u8]; L.orc_ue8m0_decode.restype = f64
            L.orc_route.argtypes = [i64, i32, i32, i32, i32, _P(f32), _P(ctypes.c_int32), _P(f64)]
            L.orc_route.restype = i32
            L.orc_route_shared.argtypes = [i64, i32, i32, i32, i32, i32, _P(f32),
                                           _P(ctypes.c_int32), _P(f64)]
            L.orc_route_shared.restype = i32
            L.orc_permute.argtypes = [i64, i32, i32] + [_P(ctypes.c_int32)] * 5
            L.orc_permute.restype = i32
            L.orc_quant_fp8_rows.argtypes = [i64, i32, _P(f64), _P(u8), _P(f32)]
            L.orc_quant_fp8_bf16_rows.argtypes = [i64, i32, _P(u16), _P(u8), _P(f32)]
            L.orc_quant_mxfp4.argtypes = [i64, i32, _P(u16), _P(u8), _P(u8)]
            L.orc_forward_bf16.argtypes = [i64, i32, i32, i32, i32, _P(u16), _P(ctypes.c_int32),
                                           _P(f64), _P(u16), _P(u16), i64, _P(i64), _P(f64), _P(u16)]
            L.orc_forward_fp8_mxfp4.argtypes = [i64, i32, i32, i32, i32, _P(u16), _P(ctypes.c_int32),
                                                _P(f64), _P(u8), _P(u8), _P(u8), _P(u8), i32, i64,
                                                _P(i64), _P(f64), _P(u16)]
            L.orc_forward_bf16_act.argtypes = [i64, i32, i32, i32, i32, i32, _P(u16),
                                               _P(ctypes.c_int32), _P(f64), _P(u16), _P(u16),
                                               i64, _P(i64), _P(f64), _P(u16)]
            L.orc_gemm1_bf16_rows.argtypes = [i32, i32, _P(u16), _P(u16), i64, _P(i64),
                                              _P(ctypes.c_int32), _P(f64)]
            L.orc_gemm1_bf16_rows_act.argtypes = [i32, i32, i32, _P(u16), _P(u16), i64, _P(i64),
                                                  _P(ctypes.c_int32), _P(f64)]
            L.orc_gemm2_bf16_rows.argtypes = [i32, i32, _P(u16), _P(u16), i64, _P(i64),
                                              _P(ctypes.c_int32), _P(f64)]
            L.orc_gemm1_fp8_rows.argtypes = [i32, i32, _P(u8), _P(f32), _P(u8), _P(u8), i32, i64,
                                             _P(i64), _P(ctypes.c_int32), _P(f64)]
            L.orc_gemm2_fp8_rows.argtypes = [i32, i32, _P(u8), _P(f32), _P(u8), _P(u8), i64,
                                             _P(i64), _P(ctypes.c_int32), _P(f64)]
            L.orc_combine.argtypes = [i32, i32, _P(u16), _P(f32), _P(ctypes.c_int32), i64, _P(i64),
                                      _P(f64), _P(u16)]
            L.orc_num_threads.restype = i32
            _lib = L
    return _lib


_CT = {np.float64: ctypes.c_double, np.float32: ctypes.c_float, np.int32: ctypes.c_int32,
       np.int64: ctypes.c_int64, np.uint8: ctypes.c_uint8, np.uint16: ctypes.c_uint16}


def _ptr(a: np.ndarray, dtype):
    assert a.dtype == dtype and a.flags.c_contiguous, (a.dtype, dtype)
    return a.ctypes.data_as(ctypes.POINTER(_CT[dtype]))


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def num_threads() -> int:
    return int(lib().orc_num_threads())


# ---- number formats ---------------------------------------------------------------

def bf16_to_f64(bits) -> np.ndarray:
    b = _c(bits, np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def f64_to_bf16(v) -> np.ndarray:
    f = lib().orc_f64_to_bf16_rne
    v = np.asarray(v, dtype=np.float64)
    return np.array([f(float(x)) for x in v.ravel()], dtype=np.uint16).reshape(v.shape)


def e4m3_decode(codes) -> np.ndarray:
    f = lib().orc_e4m3_decode
    c = np.asarray(codes, dtype=np.uint8)
    return np.array([f(int(x)) for x in c.ravel()], dtype=np.float64).reshape(c.shape)


def e4m3_encode(v) -> np.ndarray:
    f = lib().orc_e4m3_encode_rne_satfinite
    v = np.asarray(v, dtype=np.float64)
    return np.array([f(float(x)) for x in v.ravel()], dtype=np.uint8).reshape(v.shape)


def e2m1_decode(codes) -> np.ndarray:
    f = lib().orc_e2m1_decode
    c = np.asarray(codes, dtype=np.uint8)
    return np.array([f(int(x)) for x in c.ravel()], dtype=np.float64).reshape(c.shape)


def e2m1_encode(v) -> np.ndarray:
    f = lib().orc_e2m1_encode_rne_satfinite
    v = np.asarray(v, dtype=np.float64)
    return np.array([f(float(x)) for x in v.ravel()], dtype=np.uint8).reshape(v.shape)


def ue8m0_decode(b) -> np.ndarray:
    f = lib().orc_ue8m0_decode
    c = np.asarray(b, dtype=np.uint8)
    return np.array([f(int(x)) for x in c.ravel()], dtype=np.float64).reshape(c.shape)


# ---- routing, histogram, permutation ------------------------------------------------

SOFTMAX, SIGMOID = 0, 1


def route(logits: np.ndarray, k: int, score: int = SOFTMAX, renorm: bool = True,
          n_shared: int = 0):
    """Top-k by descending logit (ties to the lower index) and the slot weights (fp64);
    with n_shared > 0, slots k.. hold the shared experts E.. with weight 1."""
    lg = _c(logits, np.float32)
    T, E = lg.shape
    ids = np.empty((T, k + n_shared), np.int32)
    w = np.empty((T, k + n_shared), np.float64)
    if n_shared:
        rc = lib().orc_route_shared(T, E, k, n_shared, score, int(bool(renorm)),
                                    _ptr(lg, np.float32), _ptr(ids, np.int32),
                                    _ptr(w, np.float64))
    else:
        rc = lib().orc_route(T, E, k, score, int(bool(renorm)), _ptr(lg, np.float32),
                             _ptr(ids, np.int32), _ptr(w, np.float64))
    if rc != 0:
        raise ValueError("orc_route: bad arguments")
    return ids, w


def permute(ids: np.ndarray, E: int):
    """Per-expert histogram, exclusive prefix sum and stable scatter."""
    ids = _c(ids, np.int32)
    T, k = ids.shape
    R = T * k
    counts = np.empty(E, np.int32)
    offsets = np.empty(E + 1, np.int32)
    r2a = np.empty(R, np.int32)
    a2r = np.empty(R, np.int32)
    rc = lib().orc_permute(T, E, k, _ptr(ids, np.int32), _ptr(counts, np.int32),
                           _ptr(offsets, np.int32), _ptr(r2a, np.int32), _ptr(a2r, np.int32))
    if rc != 0:
        raise ValueError("orc_permute: expert id out of range")
    return counts, offsets, r2a, a2r


# ---- quantisers ---------------------------------------------------------------------

def quant_fp8(v: np.ndarray):
    """1x128 e4m3 codes + power-of-two fp32 scales of fp64 rows."""
    v = _c(v, np.float64)
    rows, cols = v.shape
    assert cols % 128 == 0
    codes = np.empty((rows, cols), np.uint8)
    scales = np.empty((rows, cols // 128), np.float32)
    lib().orc_quant_fp8_rows(rows, cols, _ptr(v, np.float64), _ptr(codes, np.uint8),
                             _ptr(scales, np.float32))
    return codes, scales


def quant_fp8_bf16(x_bits: np.ndarray):
    """The activation quantiser applied to bf16 rows (given as uint16 bit patterns)."""
    x = _c(x_bits, np.uint16)
    rows, cols = x.shape
    assert cols % 128 == 0
    codes = np.empty((rows, cols), np.uint8)
    scales = np.empty((rows, cols // 128), np.float32)
    lib().orc_quant_fp8_bf16_rows(rows, cols, _ptr(x, np.uint16), _ptr(codes, np.uint8),
                                  _ptr(scales, np.float32))
    return codes, scales


def quant_mxfp4(w_bits: np.ndarray):
    """MXFP4 codes (2 per byte, low nibble = even K) and UE8M0 K32 scale bytes of bf16
    rows; leading dimensions are flattened into rows."""
    w = _c(w_bits, np.uint16)
    K = w.shape[-1]
    assert K % 32 == 0
    rows = int(np.prod(w.shape[:-1]))
    packed = np.zeros(w.shape[:-1] + (K // 2,), np.uint8)
    sf = np.empty(w.shape[:-1] + (K // 32,), np.uint8)
    lib().orc_quant_mxfp4(rows, K, _ptr(w, np.uint16), _ptr(packed, np.uint8), _ptr(sf, np.uint8))
    return packed, sf


def mxfp4_dequant(packed: np.ndarray, sf: np.ndarray) -> np.ndarray:
    """fp64 values of MXFP4 weights (for tests that need the real values)."""
    lo = packed & 0xF
    hi = packed >> 4
    codes = np.stack([lo, hi], axis=-1).reshape(packed.shape[:-1] + (packed.shape[-1] * 2,))
    table = e2m1_decode(np.arange(16, dtype=np.uint8))
    scale = ue8m0_decode(np.arange(256, dtype=np.uint8))
    return table[codes] * np.repeat(scale[sf], 32, axis=-1)


# ---- expert MLP and combine ----------------------------------------------------------

def _toklist(tokens, T):
    if tokens is None:
        tokens = np.arange(T)
    return _c(tokens, np.int64)


ACTS = {"swiglu": 0, "relu2": 1}


def forward_bf16(x_bits, ids, w, w13_bits, w2_bits, tokens=None, act="swiglu"):
    """out[n] = sum_j w[t,j] * act_e(x_t).Wd^T for t = tokens[n], with act_e =
    silu(x.Wg^T) * (x.Wu^T) (W13 [E, 2I, H]) or max(x.W1^T, 0)^2 (relu2, W1 [E, I, H])."""
    x = _c(x_bits, np.uint16); ids = _c(ids, np.int32); w = _c(w, np.float64)
    w13 = _c(w13_bits, np.uint16); w2 = _c(w2_bits, np.uint16)
    T, H = x.shape
    E, rows, H2 = w13.shape
    I = rows if act == "relu2" else rows // 2
    assert H2 == H and w2.shape == (E, H, I)
    k = ids.shape[1]
    tok = _toklist(tokens, T)
    out = np.empty((len(tok), H), np.float64)
    ob = np.empty((len(tok), H), np.uint16)
    lib().orc_forward_bf16_act(T, H, I, E, k, ACTS[act], _ptr(x, np.uint16),
                               _ptr(ids, np.int32), _ptr(w, np.float64), _ptr(w13, np.uint16),
                               _ptr(w2, np.uint16), len(tok), _ptr(tok, np.int64),
                               _ptr(out, np.float64), _ptr(ob, np.uint16))
    return out, ob


def forward_fp8_mxfp4(x_bits, ids, w, w13p, w13sf, w2p, w2sf, tokens=None, requant_act=True):
    """Block-scaled forward: x -> 1x128 e4m3, GEMM1 on MXFP4, SwiGLU, act -> 1x128
    e4m3 (when requant_act), GEMM2 on MXFP4, weighted combine."""
    x = _c(x_bits, np.uint16); ids = _c(ids, np.int32); w = _c(w, np.float64)
    w13p = _c(w13p, np.uint8); w13sf = _c(w13sf, np.uint8)
    w2p = _c(w2p, np.uint8); w2sf = _c(w2sf, np.uint8)
    T, H = x.shape
    E, twoI, Hh = w13p.shape
    assert Hh * 2 == H
    I = twoI // 2
    assert w2p.shape == (E, H, I // 2)
    k = ids.shape[1]
    tok = _toklist(tokens, T)
    out = np.empty((len(tok), H), np.float64)
    ob = np.empty((len(tok), H), np.uint16)
    lib().orc_forward_fp8_mxfp4(T, H, I, E, k, _ptr(x, np.uint16), _ptr(ids, np.int32),
                                _ptr(w, np.float64), _ptr(w13p, np.uint8), _ptr(w13sf, np.uint8),
                                _ptr(w2p, np.uint8), _ptr(w2sf, np.uint8), int(bool(requant_act)),
                                len(tok), _ptr(tok, np.int64), _ptr(out, np.float64),
                                _ptr(ob, np.uint16))
    return out, ob


def gemm1_bf16_rows(x_bits, w13_bits, tok, expert, act="swiglu"):
    x = _c(x_bits, np.uint16); w13 = _c(w13_bits, np.uint16)
    tok = _c(tok, np.int64); ex = _c(expert, np.int32)
    H = x.shape[1]; I = w13.shape[1] if act == "relu2" else w13.shape[1] // 2
    out = np.empty((len(tok), I), np.float64)
    lib().orc_gemm1_bf16_rows_act(ACTS[act], H, I, _ptr(x, np.uint16), _ptr(w13, np.uint16),
                                  len(tok), _ptr(tok, np.int64), _ptr(ex, np.int32),
                                  _ptr(out, np.float64))
    return out


def gemm2_bf16_rows(a_bits, w2_bits, rows, expert):
    a = _c(a_bits, np.uint16); w2 = _c(w2_bits, np.uint16)
    rows = _c(rows, np.int64); ex = _c(expert, np.int32)
    E, H, I = w2.shape
    y = np.empty((len(rows), H), np.float64)
    lib().orc_gemm2_bf16_rows(H, I, _ptr(a, np.uint16), _ptr(w2, np.uint16), len(rows),
                              _ptr(rows, np.int64), _ptr(ex, np.int32), _ptr(y, np.float64))
    return y


def gemm1_fp8_rows(xq, sx, w13p, w13sf, tok, expert, requant_act=True):
    xq = _c(xq, np.uint8); sx = _c(sx, np.float32)
    w13p = _c(w13p, np.uint8); w13sf = _c(w13sf, np.uint8)
    tok = _c(tok, np.int64); ex = _c(expert, np.int32)
    H = xq.shape[1]; I = w13p.shape[1] // 2
    act = np.empty((len(tok), I), np.float64)
    lib().orc_gemm1_fp8_rows(H, I, _ptr(xq, np.uint8), _ptr(sx, np.float32), _ptr(w13p, np.uint8),
                             _ptr(w13sf, np.uint8), int(bool(requant_act)), len(tok),
                             _ptr(tok, np.int64), _ptr(ex, np.int32), _ptr(act, np.float64))
    return act


def gemm2_fp8_rows(aq, sa, w2p, w2sf, rows, expert):
    aq = _c(aq, np.uint8); sa = _c(sa, np.float32)
    w2p = _c(w2p, np.uint8); w2sf = _c(w2sf, np.uint8)
    rows = _c(rows, np.int64); ex = _c(expert, np.int32)
    E, H, Ih = w2p.shape
    I = Ih * 2
    y = np.empty((len(rows), H), np.float64)
    lib().orc_gemm2_fp8_rows(H, I, _ptr(aq, np.uint8), _ptr(sa, np.float32), _ptr(w2p, np.uint8),
                             _ptr(w2sf, np.uint8), len(rows), _ptr(rows, np.int64),
                             _ptr(ex, np.int32), _ptr(y, np.float64))
    return y


def combine(y_bits, w, assign2row, tokens=None):
    y = _c(y_bits, np.uint16); w = _c(w, np.float32); a2r = _c(assign2row, np.int32)
    T, k = w.shape
    H = y.shape[1]
    tok = _toklist(tokens, T)
    out = np.empty((len(tok), H), np.float64)
    ob = np.empty((len(tok), H), np.uint16)
    lib().orc_combine(H, k, _ptr(y, np.uint16), _ptr(w, np.float32), _ptr(a2r, np.int32),
                      len(tok), _ptr(tok, np.int64), _ptr(out, np.float64), _ptr(ob, np.uint16))
    return out, ob
