"""Parity of the CUDA path (through the C ABI) with the fp64 CPU oracle.

Indices (routing ids, counts, offsets, row2assign, assign2row) must be bit-exact; floating
point outputs must meet max|err| <= 2e-2 * max|ref| and cosine >= 0.9999.  Every output
buffer carries a canary tail that must survive (out-of-bounds stores)."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import (COS_BF16, assert_close, canary_intact, dev, f64, gpu_permute, gpu_route,
                      oracle_route, to_dev_i32, with_canary, workspace)
from mixture_experts_routed_histogram_b200 import _capi as C
from mixture_experts_routed_histogram_b200 import inputs as I

pytestmark = pytest.mark.gpu

W = I.WORKLOADS

# Small shapes that span several tiles and ragged tails on every GEMM edge.
SMALL = {
    "tiny": W["tiny"],
    "odd_h384_i192": I.Workload("odd", 129, 384, 192, 4, 2),          # I % 128 = 64, H % 256 != 0
    "one_token": I.Workload("one", 1, 256, 128, 8, 2),
    "seven_tokens_e512_k10": I.Workload("e512", 7, 256, 128, 512, 10, routing="uniform"),
    "sigmoid_top1": I.Workload("sig", 200, 512, 256, 16, 1, score="sigmoid", renorm=False),
    "zipf_empty_experts": I.Workload("zipf", 96, 512, 384, 8, 2, routing="zipf"),
    "many_tiles": I.Workload("many", 1000, 512, 256, 8, 4),
    # ReLU2 (non-gated, W1 [E, I, H]): one partial 256-column tile (I = 192), two and a
    # half tiles (I = 640), and a decode-sized batch (GEMM2 on the decode kernels)
    "relu2_i192": I.Workload("r2a", 300, 256, 192, 8, 2, act="relu2"),
    "relu2_i640": I.Workload("r2b", 1000, 512, 640, 8, 4, act="relu2"),
    "relu2_t48": I.Workload("r2c", 48, 512, 256, 8, 2, act="relu2"),
    # shared experts: experts E.. on every token with weight 1 (decode-sized and large)
    "shared1_t40": I.Workload("sh1", 40, 256, 128, 8, 2, n_shared=1),
    "shared2_t500": I.Workload("sh2", 500, 512, 256, 16, 4, n_shared=2),
    # decode-sized with K split into slices: GEMM2 picks the count from its busy tiles
    # (2 for I = 3072; 4-6 of up to 7 for I = 10752, 168 K blocks); GEMM1 splits H = 1024 in 2
    "ksplit_i3072": I.Workload("ks2", 24, 512, 3072, 4, 2, routing="zipf"),
    "ksplit_h1024_i10752": I.Workload("ks7", 8, 1024, 10752, 4, 2),
}


def _skewed_logits(wl, x):
    lg = I.make_logits(wl, x)
    lg[:, 3] += 100.0  # every token's top-1 is expert 3
    return lg


# ------------------------------------------------------------------ routing / permutation

ROUTE_CASES = {
    "tiny": W["tiny"],
    "qwen3_30b_a3b": W["qwen3_30b_a3b"],
    "llama4_scout": W["llama4_scout"],
    "fp8_mxfp4_T16384": W["fp8_mxfp4"].with_T(16384),
    "decode_T256": W["decode"].with_T(256),
    "e1000_k32": I.Workload("wide", 300, 256, 128, 1000, 32),
    "e16_k4_shared2": I.Workload("shr", 300, 256, 128, 16, 4, n_shared=2),
    "e8_k2_shared1_t40": I.Workload("shs", 40, 256, 128, 8, 2, n_shared=1),
}


@pytest.mark.parametrize("name", list(ROUTE_CASES))
def test_route_and_permute_bitexact(name):
    wl = ROUTE_CASES[name]
    x = I.make_x(wl, 0, dev())
    lg = I.make_logits(wl, x)
    if name == "tiny":   # coarse logits: many exact ties
        lg = torch.round(lg * 2) / 2
    shape = C.MoeShape.from_workload(wl)
    ids, w = gpu_route(shape, lg)
    oids, ow = oracle_route(wl, lg)
    assert np.array_equal(ids.cpu().numpy(), oids)
    assert np.allclose(w.cpu().numpy(), ow, rtol=2e-6, atol=2e-7)
    ws = workspace(shape)
    # permutation of the oracle's ids (an input independent of the CUDA path)
    counts, offsets, r2a, a2r = gpu_permute(shape, to_dev_i32(oids), ws)
    oc, oo, or2a, oa2r = oracle.permute(oids, wl.E_all)
    assert np.array_equal(counts.cpu().numpy(), oc)
    assert np.array_equal(offsets.cpu().numpy(), oo)
    assert np.array_equal(r2a.cpu().numpy(), or2a)
    assert np.array_equal(a2r.cpu().numpy(), oa2r)
    assert C.moe_get_device_status(ws) == 0


@pytest.mark.parametrize("R,E", [(1, 1), (5, 8), (2048, 4), (2049, 300), (163840, 512),
                                 (65536, 128), (600000, 64)])
def test_permute_random_ids_bitexact(R, E):
    rng = np.random.default_rng(R + E)
    ids = rng.integers(0, E, R).astype(np.int32)
    if E >= 8:
        ids[rng.random(R) < 0.5] = 3             # heavy skew
    shape = C.MoeShape.of(R, 64, 64, E, 1)
    ws = workspace(shape)
    counts, offsets, r2a, a2r = gpu_permute(shape, to_dev_i32(ids.reshape(R, 1)), ws)
    oc, oo, or2a, oa2r = oracle.permute(ids.reshape(R, 1), E)
    assert np.array_equal(counts.cpu().numpy(), oc)
    assert np.array_equal(offsets.cpu().numpy(), oo)
    assert np.array_equal(r2a.cpu().numpy(), or2a)
    assert np.array_equal(a2r.cpu().numpy(), oa2r)


def test_permute_flags_bad_ids():
    shape = C.MoeShape.of(4, 64, 64, 8, 1)
    ws = workspace(shape)
    gpu_permute(shape, to_dev_i32(np.array([[0], [8], [1], [2]])), ws)
    assert C.moe_get_device_status(ws) == C.MOE_ERR_DEVICE_BAD_INDEX
    assert C.moe_get_device_status(ws) == 0  # read clears it


# ------------------------------------------------------------------ GEMM stages

def _stage_inputs(wl, skew=False):
    inp = I.make_inputs(wl, 0, dev())
    lg = _skewed_logits(wl, inp["x"]) if skew else inp["logits"]
    oids, ow = oracle_route(wl, lg)
    oc, oo, or2a, oa2r = oracle.permute(oids, wl.E_all)
    return inp, oids, ow, oo, or2a, oa2r


GEMM_CASES = dict(SMALL)
GEMM_CASES["skew_one_expert"] = I.Workload("skew", 300, 256, 128, 8, 1)


@pytest.mark.parametrize("name", list(GEMM_CASES))
def test_gemm1_swiglu_parity(name):
    wl = GEMM_CASES[name]
    inp, oids, ow, oo, or2a, oa2r = _stage_inputs(wl, skew=name.startswith("skew"))
    shape = C.MoeShape.from_workload(wl)
    ws = workspace(shape)
    R = wl.R
    buf, act = with_canary(R, wl.I)
    C.moe_grouped_gemm1_swiglu(shape, inp["x"], None, to_dev_i32(or2a), to_dev_i32(oo),
                               inp["w13"], None, act, None, ws)
    torch.cuda.synchronize()
    assert C.moe_get_device_status(ws) == 0
    assert canary_intact(buf, R, wl.I)
    tok = or2a.astype(np.int64) // (wl.k + wl.n_shared)
    ex = np.repeat(np.arange(wl.E_all), np.diff(oo)).astype(np.int32)
    ref = oracle.gemm1_bf16_rows(I.bits(inp["x"]), I.bits(inp["w13"]), tok, ex, act=wl.act)
    assert_close(f64(act), ref, what=f"gemm1 {name}")


@pytest.mark.parametrize("name", list(GEMM_CASES))
def test_gemm2_parity(name):
    wl = GEMM_CASES[name]
    inp, oids, ow, oo, or2a, oa2r = _stage_inputs(wl, skew=name.startswith("skew"))
    shape = C.MoeShape.from_workload(wl)
    ws = workspace(shape)
    R = wl.R
    g = torch.Generator(device=dev()).manual_seed(5)
    act = torch.randn(R, wl.I, generator=g, device=dev()).to(torch.bfloat16)
    buf, y = with_canary(R, wl.H)
    C.moe_grouped_gemm2(shape, act, None, to_dev_i32(oo), inp["w2"], None, y, ws)
    torch.cuda.synchronize()
    assert C.moe_get_device_status(ws) == 0
    assert canary_intact(buf, R, wl.H)
    ex = np.repeat(np.arange(wl.E_all), np.diff(oo)).astype(np.int32)
    ref = oracle.gemm2_bf16_rows(I.bits(act), I.bits(inp["w2"]), np.arange(R), ex)
    assert_close(f64(y), ref, what=f"gemm2 {name}")


@pytest.mark.parametrize("name", ["tiny", "odd_h384_i192", "seven_tokens_e512_k10"])
def test_combine_parity(name):
    wl = SMALL[name]
    inp, oids, ow, oo, or2a, oa2r = _stage_inputs(wl)
    shape = C.MoeShape.from_workload(wl)
    g = torch.Generator(device=dev()).manual_seed(6)
    y = torch.randn(wl.R, wl.H, generator=g, device=dev()).to(torch.bfloat16)
    w32 = ow.astype(np.float32)
    buf, out = with_canary(wl.T, wl.H)
    C.moe_combine(shape, y, torch.from_numpy(w32).to(dev()), to_dev_i32(oa2r), out)
    torch.cuda.synchronize()
    assert canary_intact(buf, wl.T, wl.H)
    ref, refb = oracle.combine(I.bits(y), w32, oa2r)
    got = f64(out)
    # one fp32 sum of k terms, one bf16 rounding: within one bf16 ulp of the oracle
    assert np.all(np.abs(got - ref) <= np.abs(ref) * 2.0 ** -7 + 1e-30)


# ------------------------------------------------------------------ whole forward pass

def _forward(wl, inp, logits, ws):
    shape = C.MoeShape.from_workload(wl)
    buf, out = with_canary(wl.T, wl.H)
    ids = torch.empty(wl.T, wl.k + wl.n_shared, dtype=torch.int32, device=dev())
    C.moe_forward(shape, inp["x"], logits, inp["w13"], None, inp["w2"], None, out, ids, ws)
    torch.cuda.synchronize()
    assert canary_intact(buf, wl.T, wl.H)
    return out, ids


def _check_forward(wl, inp, logits, tokens, skew=False):
    shape = C.MoeShape.from_workload(wl)
    ws = workspace(shape)
    out, ids = _forward(wl, inp, logits, ws)
    assert C.moe_get_device_status(ws) == 0
    oids, ow = oracle_route(wl, logits)
    assert np.array_equal(ids.cpu().numpy(), oids)
    ref, _ = oracle.forward_bf16(I.bits(inp["x"]), oids, ow, I.bits(inp["w13"]),
                                 I.bits(inp["w2"]), tokens, act=wl.act)
    got = f64(out)[tokens]
    return assert_close(got, ref, COS_BF16, what=f"forward {wl.name} T={wl.T}"), (out, ws)


@pytest.mark.parametrize("name", list(SMALL))
def test_forward_small_parity(name):
    wl = SMALL[name]
    inp = I.make_inputs(wl, 0, dev())
    _check_forward(wl, inp, inp["logits"], np.arange(wl.T))


def test_forward_skewed_one_expert():
    wl = I.Workload("skew", 300, 256, 128, 8, 1)
    inp = I.make_inputs(wl, 0, dev())
    _check_forward(wl, inp, _skewed_logits(wl, inp["x"]), np.arange(wl.T))


@pytest.mark.parametrize("wl", [I.Workload("ties", 300, 256, 128, 64, 4),
                                I.Workload("wide", 100, 256, 128, 1000, 32, routing="uniform")],
                         ids=["ties_e64_k4", "e1000_k32"])
def test_forward_front_end_ties_and_wide_routing(wl):
    """The large-batch front end of moe_forward (routing fused with the chunk histograms,
    scan, scatter): coarse logits with many exact ties, and 1000 experts with top-32."""
    inp = I.make_inputs(wl, 0, dev())
    lg = inp["logits"]
    if wl.name == "ties":
        lg = torch.round(lg * 2) / 2
    _check_forward(wl, inp, lg, np.arange(wl.T))


def test_forward_deterministic():
    wl = SMALL["many_tiles"]
    inp = I.make_inputs(wl, 0, dev())
    shape = C.MoeShape.from_workload(wl)
    ws = workspace(shape)
    a, _ = _forward(wl, inp, inp["logits"], ws)
    b, _ = _forward(wl, inp, inp["logits"], ws)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


FULL = {
    "qwen3_30b_a3b": W["qwen3_30b_a3b"],
    "llama4_scout": W["llama4_scout"],
    **{f"decode_T{t}": W["decode"].with_T(t) for t in I.DECODE_T_SWEEP},
    # points of the parameter grid: 8192 rows per expert (top-1), 512 (E=128, top-8) and
    # 2048 at H=I=4096 -- single-SM and SM-pair GEMM2, K up to 4096
    **{n: W[n] for n in ("grid_d2048_e8_k1", "grid_d2048_e128_k8", "grid_d4096_e16_k4")},
    "nemotron_relu2": W["nemotron_relu2"],
    "qwen3_30b_a3b_shared1": W["qwen3_30b_a3b_shared1"],
}


@pytest.mark.parametrize("name", list(FULL))
def test_forward_full_size_parity(name):
    """Full-size workloads in the launch configuration the benchmark times; the oracle
    checks a seeded token subset (always including the first and last token)."""
    wl = FULL[name]
    inp = I.make_inputs(wl, 0, dev())
    n = 64 if wl.name == "decode" else 256
    _check_forward(wl, inp, inp["logits"], I.parity_tokens(wl.T, n))


# Expert row counts that put an expert's last token chunk (of up to 256 rows, padded to a
# multiple of 16) on every boundary: 1, 15-17, 31-33 rows, exactly one and two chunks, one
# row more or less, experts of three to seven chunks (767 .. 1537), and empty experts
# between them; and last chunks of 17-65 rows after two or three full ones (273 .. 788).
CHUNK_COUNTS = [1, 0, 15, 16, 17, 31, 32, 33, 0, 255, 256, 257, 511, 512, 513, 8,
                767, 768, 769, 1024, 1025, 1537, 273, 530, 545, 576, 577, 788]


def _chunk_ids():
    ids = np.repeat(np.arange(len(CHUNK_COUNTS), dtype=np.int32), CHUNK_COUNTS)
    rng = np.random.default_rng(11)
    return rng.permutation(ids).reshape(-1, 1)        # k = 1: one slot per token


@pytest.mark.parametrize("H,Iw,act", [(256, 128, "swiglu"), (384, 192, "swiglu"),
                                     (512, 320, "relu2")])
def test_gemms_on_chunk_boundaries(H, Iw, act):
    ids = _chunk_ids()
    T, E = ids.shape[0], len(CHUNK_COUNTS)
    wl = I.Workload("chunks", T, H, Iw, E, 1, act=act)
    inp = I.make_inputs(wl, 0, dev())
    oc, oo, or2a, oa2r = oracle.permute(ids, E)
    assert list(oc) == CHUNK_COUNTS
    shape = C.MoeShape.from_workload(wl)
    ws = workspace(shape)
    R = wl.R
    buf, act_t = with_canary(R, Iw)
    C.moe_grouped_gemm1_swiglu(shape, inp["x"], None, to_dev_i32(or2a), to_dev_i32(oo),
                               inp["w13"], None, act_t, None, ws)
    buf2, y = with_canary(R, H)
    g = torch.Generator(device=dev()).manual_seed(5)
    a2 = torch.randn(R, Iw, generator=g, device=dev()).to(torch.bfloat16)
    C.moe_grouped_gemm2(shape, a2, None, to_dev_i32(oo), inp["w2"], None, y, ws)
    torch.cuda.synchronize()
    assert C.moe_get_device_status(ws) == 0
    assert canary_intact(buf, R, Iw) and canary_intact(buf2, R, H)
    tok = or2a.astype(np.int64)
    ex = np.repeat(np.arange(E), np.diff(oo)).astype(np.int32)
    ref1 = oracle.gemm1_bf16_rows(I.bits(inp["x"]), I.bits(inp["w13"]), tok, ex, act=act)
    assert_close(f64(act_t), ref1, what=f"gemm1 chunks {act}")
    ref2 = oracle.gemm2_bf16_rows(I.bits(a2), I.bits(inp["w2"]), np.arange(R), ex)
    assert_close(f64(y), ref2, what="gemm2 chunks")
    # every row separately: a tile that wrote another expert's rows would show here
    got1 = f64(act_t)
    for e in range(E):
        lo, hi = oo[e], oo[e + 1]
        if hi > lo:
            assert_close(got1[lo:hi], ref1[lo:hi], what=f"gemm1 expert {e}")
