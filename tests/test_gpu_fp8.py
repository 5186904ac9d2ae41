"""Parity of the block-scaled path (FP8 e4m3 activations x MXFP4 weights) with the oracle.

Quantisers: bit-exact codes and scales.  GEMM1: the requantised activation against the
exact (fp64, not requantised) SwiGLU output, within half an e4m3 step plus the scale's
subnormal step.  GEMM2 and the forward pass: max|err| <= 2e-2 * max|ref| and cosine
>= 0.999 (0.9999 where both sides consume identical quantised inputs)."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import (COS_BF16, COS_FP8, assert_close, canary_intact, dev, f64, oracle_route,
                      to_dev_i32, with_canary, workspace)
from mixture_experts_routed_histogram_b200 import _capi as C
from mixture_experts_routed_histogram_b200 import inputs as I

pytestmark = pytest.mark.gpu

W = I.WORKLOADS


def _np(t):
    return t.detach().cpu().numpy()


# ------------------------------------------------------------------ quantisers

@pytest.mark.parametrize("T,H", [(64, 256), (1024, 2560), (3, 128)])
def test_quantize_x_bitexact(T, H):
    wl = I.Workload("q", T, H, 128, 4, 2, dtype="fp8_mxfp4")
    x = I.make_x(wl, 0, dev())
    if T >= 3:                       # edge groups: all zero, huge, tiny, negative tiny
        x[0, :128] = 0
        x[1, :128] = torch.linspace(-3e4, 3e4, 128, device=dev()).to(torch.bfloat16)
        x[2, :128] = (torch.randn(128, device=dev()) * 1e-30).to(torch.bfloat16)
    shape = C.MoeShape.from_workload(wl)
    xq = torch.empty(T, H, dtype=torch.uint8, device=dev())
    sx = torch.empty(T, H // 128, dtype=torch.float32, device=dev())
    C.moe_quantize_x(shape, x, xq, sx)
    torch.cuda.synchronize()
    codes, scales = oracle.quant_fp8_bf16(I.bits(x))
    assert np.array_equal(_np(sx), scales)
    assert np.array_equal(_np(xq), codes)


@pytest.mark.parametrize("rows,K", [(1280 * 2, 2560), (2560, 640), (7, 64)])
def test_quantize_weights_mxfp4_bitexact(rows, K):
    g = torch.Generator(device=dev()).manual_seed(rows + K)
    w = (torch.randn(rows, K, generator=g, device=dev()) / K ** 0.5).to(torch.bfloat16)
    w[0, :32] = 0                                      # amax = 0 block
    w[1, :32] = 5.0                                    # exact ties / saturation
    w[1, 1] = 0.75 * 4
    packed = torch.empty(rows, K // 2, dtype=torch.uint8, device=dev())
    sf = torch.empty(rows, K // 32, dtype=torch.uint8, device=dev())
    C.moe_quantize_weights_mxfp4(w, packed, sf)
    torch.cuda.synchronize()
    op, osf = oracle.quant_mxfp4(I.bits(w))
    assert np.array_equal(_np(sf), osf)
    assert np.array_equal(_np(packed), op)


# ------------------------------------------------------------------ GEMM stages

SMALL = {
    "e8_h256_i128": I.Workload("s1", 64, 256, 128, 8, 2, dtype="fp8_mxfp4"),
    "e512_k10_t7": I.Workload("s2", 7, 256, 256, 512, 10, dtype="fp8_mxfp4", routing="uniform"),
    "ragged_t129_h384": I.Workload("s3", 129, 384, 256, 4, 2, dtype="fp8_mxfp4"),
    "fp8_shape_t64": W["fp8_mxfp4"].with_T(64),
    # > 48 rows per expert: the single-SM block-scaled kernels, 5 and 8 K blocks in GEMM2
    "e8_t300_i640": I.Workload("s4", 300, 256, 640, 8, 2, dtype="fp8_mxfp4"),
    "e4_t200_i1024": I.Workload("s5", 200, 256, 1024, 4, 2, dtype="fp8_mxfp4"),
}


def _routing(wl, inp):
    oids, ow = oracle_route(wl, inp["logits"])
    oc, oo, or2a, oa2r = oracle.permute(oids, wl.E_all)
    return oids, ow, oo, or2a, oa2r


@pytest.mark.parametrize("name", list(SMALL))
def test_gemm1_fp8_parity(name):
    wl = SMALL[name]
    inp = I.make_inputs(wl, 0, dev())
    oids, ow, oo, or2a, oa2r = _routing(wl, inp)
    shape = C.MoeShape.from_workload(wl)
    ws = workspace(shape)
    xq_np, sx_np = oracle.quant_fp8_bf16(I.bits(inp["x"]))
    xq = torch.from_numpy(xq_np).to(dev())
    sx = torch.from_numpy(sx_np).to(dev())
    R = wl.R
    act = torch.empty(R * wl.I + 512, dtype=torch.uint8, device=dev()).fill_(0x5A)
    act_sf = torch.empty(R, wl.I // 128, dtype=torch.float32, device=dev())
    C.moe_grouped_gemm1_swiglu(shape, xq, sx, to_dev_i32(or2a), to_dev_i32(oo), inp["w13"],
                               inp["w13_sf"], act, act_sf, ws)
    torch.cuda.synchronize()
    assert C.moe_get_device_status(ws) == 0
    assert bool((act[R * wl.I:] == 0x5A).all())
    tok = or2a.astype(np.int64) // (wl.k + wl.n_shared)
    ex = np.repeat(np.arange(wl.E_all), np.diff(oo)).astype(np.int32)
    exact = oracle.gemm1_fp8_rows(xq_np, sx_np, _np(inp["w13"]), _np(inp["w13_sf"]), tok, ex,
                                  requant_act=False)
    scales = np.repeat(_np(act_sf).astype(np.float64), 128, axis=1)
    got = oracle.e4m3_decode(_np(act[:R * wl.I]).reshape(R, wl.I)) * scales
    # every code is within half an e4m3 step (2^-4 relative) of the exact value, or within
    # half the smallest subnormal step (2^-10 of the scale) near zero
    bound = np.abs(exact) * 2.0 ** -4 * (1 + 1e-3) + scales * 2.0 ** -10 + 1e-6 * np.abs(exact).max()
    bad = np.abs(got - exact) > bound
    assert not bad.any(), f"{bad.sum()} of {bad.size} act codes off by more than half a step"
    # e4m3 keeps 4 significant bits, so the requantised activation itself is only good to
    # half a step (2^-4 of max|ref|); the 2e-2 bar applies to the layer output
    assert_close(got, exact, COS_FP8, rel=2.0 ** -4 * 1.01, what=f"gemm1 fp8 {name}")


@pytest.mark.parametrize("name", list(SMALL))
def test_gemm2_fp8_parity(name):
    wl = SMALL[name]
    inp = I.make_inputs(wl, 0, dev())
    oids, ow, oo, or2a, oa2r = _routing(wl, inp)
    shape = C.MoeShape.from_workload(wl)
    ws = workspace(shape)
    R = wl.R
    rng = np.random.default_rng(9)
    a64 = rng.standard_normal((R, wl.I)) * np.exp(rng.uniform(-3, 3, (R, 1)))
    aq_np, sa_np = oracle.quant_fp8(a64)
    buf, y = with_canary(R, wl.H)
    C.moe_grouped_gemm2(shape, torch.from_numpy(aq_np).to(dev()), torch.from_numpy(sa_np).to(dev()),
                        to_dev_i32(oo), inp["w2"], inp["w2_sf"], y, ws)
    torch.cuda.synchronize()
    assert C.moe_get_device_status(ws) == 0
    assert canary_intact(buf, R, wl.H)
    ex = np.repeat(np.arange(wl.E_all), np.diff(oo)).astype(np.int32)
    ref = oracle.gemm2_fp8_rows(aq_np, sa_np, _np(inp["w2"]), _np(inp["w2_sf"]), np.arange(R), ex)
    assert_close(f64(y), ref, COS_BF16, what=f"gemm2 fp8 {name}")


# ------------------------------------------------------------------ forward

def _forward_check(wl, tokens, weights_from_gpu_quantiser=False):
    inp = I.make_inputs(wl, 0, dev())
    shape = C.MoeShape.from_workload(wl)
    ws = workspace(shape)
    buf, out = with_canary(wl.T, wl.H)
    ids = torch.empty(wl.T, wl.k + wl.n_shared, dtype=torch.int32, device=dev())
    C.moe_forward(shape, inp["x"], inp["logits"], inp["w13"], inp["w13_sf"], inp["w2"],
                  inp["w2_sf"], out, ids, ws)
    torch.cuda.synchronize()
    assert C.moe_get_device_status(ws) == 0
    assert canary_intact(buf, wl.T, wl.H)
    oids, ow = oracle_route(wl, inp["logits"])
    assert np.array_equal(_np(ids), oids)
    ref, _ = oracle.forward_fp8_mxfp4(I.bits(inp["x"]), oids, ow, _np(inp["w13"]),
                                      _np(inp["w13_sf"]), _np(inp["w2"]), _np(inp["w2_sf"]),
                                      tokens, requant_act=True)
    return assert_close(f64(out)[tokens], ref, COS_FP8, what=f"fp8 forward {wl.name} T={wl.T}")


@pytest.mark.parametrize("name", list(SMALL))
def test_forward_fp8_small(name):
    wl = SMALL[name]
    _forward_check(wl, np.arange(wl.T))


@pytest.mark.parametrize("T", I.FP8_T_SWEEP)
def test_forward_fp8_full_size(T):
    """The FP8 x MXFP4 workload (H=2560, E=512, k=10, I=640) over its T sweep; the oracle
    checks a seeded 256-token subset that always includes the first and last token."""
    wl = W["fp8_mxfp4"].with_T(T)
    _forward_check(wl, I.parity_tokens(T, 256))


@pytest.mark.parametrize("T", [64, 300])
def test_forward_fp8_on_quantised_gaussian_weights(T):
    """The block-scaled forward on MXFP4 weights that the oracle's OCP MX quantiser made from
    N(0, 1/fan_in) bf16 weights (the synthetic generator draws codes and scale bytes
    directly, with a narrower spread of scales): both sides consume the same codes."""
    wl16 = I.Workload("qg", T, 256, 256, 8, 2)
    wl = I.Workload("qg", T, 256, 256, 8, 2, dtype="fp8_mxfp4")
    x = I.make_x(wl16, 0, "cpu")
    logits = I.make_logits(wl16, x)
    w13_bf, w2_bf = I.make_weights(wl16, 0, "cpu")
    w13p, w13sf = oracle.quant_mxfp4(I.bits(w13_bf))
    w2p, w2sf = oracle.quant_mxfp4(I.bits(w2_bf))
    # scale bytes as gaussian blocks give them (three values here) and codes that are not
    # drawn from the generator's table
    assert len(np.unique(w13sf)) >= 3 and len(np.unique(w2sf)) >= 3
    shape = C.MoeShape.from_workload(wl)
    ws = workspace(shape)
    buf, out = with_canary(T, wl.H)
    d = {n: torch.from_numpy(np.ascontiguousarray(a)).to(dev())
         for n, a in (("w13", w13p), ("w13_sf", w13sf), ("w2", w2p), ("w2_sf", w2sf))}
    C.moe_forward(shape, x.to(dev()), logits.to(dev()), d["w13"], d["w13_sf"], d["w2"],
                  d["w2_sf"], out, None, ws)
    torch.cuda.synchronize()
    assert C.moe_get_device_status(ws) == 0
    assert canary_intact(buf, T, wl.H)
    oids, ow = oracle_route(wl, logits)
    ref, _ = oracle.forward_fp8_mxfp4(I.bits(x), oids, ow, w13p, w13sf, w2p, w2sf,
                                      np.arange(T), requant_act=True)
    assert_close(f64(out), ref, COS_FP8, what=f"fp8 forward on quantised gaussian weights T={T}")
