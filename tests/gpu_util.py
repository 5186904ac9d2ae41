"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI binding and
compare it with the CPU oracle."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from mixture_experts_routed_histogram_b200 import _capi as C
from mixture_experts_routed_histogram_b200 import inputs as I

SENTINEL = 0x7E7E  # canary pattern written past the end of every output buffer

# Acceptance bars: BF16 output max|err| <= 2e-2 * max|ref| and cosine >= 0.9999
# (>= 0.999 for the block-scaled path); indices bit-exact.
REL_MAX = 2e-2
COS_BF16 = 0.9999
COS_FP8 = 0.999


def dev():
    return torch.device("cuda", 0)


def workspace(shape):
    n = C.moe_workspace_size(shape)
    assert n > 0
    ws = torch.empty(n, dtype=torch.uint8, device=dev())
    C.moe_workspace_init(ws)
    return ws


def with_canary(rows: int, cols: int, dtype=torch.bfloat16, extra_rows: int = 2):
    """Tensor [rows + extra_rows, cols] whose tail rows hold SENTINEL; returns (buf, view)."""
    buf = torch.empty((rows + extra_rows) * cols, dtype=torch.int16, device=dev())
    buf.fill_(SENTINEL)
    view = buf[: rows * cols].view(dtype).view(rows, cols) if dtype == torch.bfloat16 else None
    return buf, view


def canary_intact(buf, rows: int, cols: int) -> bool:
    return bool((buf[rows * cols:] == SENTINEL).all().item())


def f64(t_bf16: torch.Tensor) -> np.ndarray:
    return t_bf16.detach().float().cpu().numpy().astype(np.float64)


def assert_close(got, ref, cos_min=COS_BF16, rel=REL_MAX, what=""):
    got = np.asarray(got, np.float64).ravel()
    ref = np.asarray(ref, np.float64).ravel()
    assert got.shape == ref.shape
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = float(np.abs(got - ref).max()) if got.size else 0.0
    scale = float(np.abs(ref).max()) if ref.size else 0.0
    den = float(np.linalg.norm(got) * np.linalg.norm(ref))
    cos = float(np.dot(got, ref) / den) if den > 0 else 1.0
    assert err <= rel * scale and cos >= cos_min, \
        f"{what}: max|err|={err:.4e} max|ref|={scale:.4e} ({err / max(scale, 1e-300):.3e}) cos={cos:.8f}"
    return err / max(scale, 1e-300), cos


def routing_logits(wl: I.Workload, x: torch.Tensor, seed=0):
    return I.make_logits(wl, x, seed)


def oracle_route(wl: I.Workload, logits: torch.Tensor):
    score = oracle.SOFTMAX if wl.score == "softmax" else oracle.SIGMOID
    return oracle.route(logits.cpu().numpy(), wl.k, score, wl.renorm, n_shared=wl.n_shared)


def gpu_route(shape, logits):
    T, k = shape.T, shape.k + shape.n_shared
    ids = torch.empty(T, k, dtype=torch.int32, device=dev())
    w = torch.empty(T, k, dtype=torch.float32, device=dev())
    C.moe_route(shape, logits, ids, w)
    return ids, w


def gpu_permute(shape, ids, ws):
    R, E = shape.T * (shape.k + shape.n_shared), shape.E + shape.n_shared
    counts = torch.empty(E, dtype=torch.int32, device=dev())
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev())
    r2a = torch.empty(max(R, 1), dtype=torch.int32, device=dev())
    a2r = torch.empty(max(R, 1), dtype=torch.int32, device=dev())
    C.moe_permute(shape, ids, counts, offsets, r2a, a2r, ws)
    return counts, offsets, r2a[:R], a2r[:R]


def to_dev_i32(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, np.int32)).to(dev())
