"""Failure detection without a GPU fault: a test hook leaves one pipeline stage of a
grouped-GEMM launch unfilled, the consumer's bounded mbarrier wait (shortened to 50 ms)
expires, every role of the kernel unwinds, the status word reads MOE_ERR_DEVICE_TIMEOUT,
and the context stays usable: the same launch without the hook gives the same bits as a
clean launch made before the failure (and the first case also matches the oracle).

The shapes pick each GEMM kernel family: decode-sized (single SMs, weights on the MMA's
M = 128 side), SM pairs (weights on the M = 256 side; SwiGLU, ReLU2 and experts of several
256-row chunks), and the block-scaled FP8 x MXFP4 kernels in both their forms."""
import time

import numpy as np
import pytest
import torch

import oracle
from gpu_util import assert_close, dev, f64, oracle_route, to_dev_i32, workspace
from mixture_experts_routed_histogram_b200 import _capi as C
from mixture_experts_routed_histogram_b200 import inputs as I

pytestmark = pytest.mark.gpu

CASES = {
    "bf16_swap": I.WORKLOADS["tiny"],                                  # T <= 64
    "bf16_pairs": I.Workload("fs", 300, 256, 128, 8, 2),               # 75 rows / expert
    "bf16_pairs_relu2": I.Workload("fr", 300, 256, 128, 8, 2, act="relu2"),
    "bf16_pairs_4_chunks": I.Workload("fp", 2048, 256, 128, 2, 1),     # 1024 rows / expert
    "fp8_single_sm": I.Workload("f8", 300, 256, 256, 4, 2, dtype="fp8_mxfp4"),
    "fp8_swap": I.Workload("f8s", 64, 256, 128, 8, 2, dtype="fp8_mxfp4"),
}


def _setup(wl):
    inp = I.make_inputs(wl, 0, dev())
    oids, _ = oracle_route(wl, inp["logits"])
    _, oo, or2a, _ = oracle.permute(oids, wl.E_all)
    shape = C.MoeShape.from_workload(wl)
    ws = workspace(shape)
    fp8 = wl.dtype == "fp8_mxfp4"
    st = {"inp": inp, "oo": oo, "or2a": or2a, "shape": shape, "ws": ws, "fp8": fp8}
    if fp8:
        xq = torch.empty(wl.T, wl.H, dtype=torch.uint8, device=dev())
        sx = torch.empty(wl.T, wl.H // 128, dtype=torch.float32, device=dev())
        C.moe_quantize_x(shape, inp["x"], xq, sx)
        rng = np.random.default_rng(5)
        aq, sa = oracle.quant_fp8(rng.standard_normal((wl.R, wl.I)))
        st.update(xq=xq, sx=sx, a_in=torch.from_numpy(aq).to(dev()),
                  sa_in=torch.from_numpy(sa).to(dev()))
    else:
        g = torch.Generator(device=dev()).manual_seed(3)
        st["a_in"] = torch.randn(wl.R, wl.I, generator=g, device=dev()).to(torch.bfloat16)
        st["sa_in"] = None
    return st


def _run(wl, st, which):
    inp, shape, ws = st["inp"], st["shape"], st["ws"]
    if which == "gemm1":
        if st["fp8"]:
            act = torch.empty(wl.R, wl.I, dtype=torch.uint8, device=dev())
            act_sf = torch.empty(wl.R, wl.I // 128, dtype=torch.float32, device=dev())
            C.moe_grouped_gemm1_swiglu(shape, st["xq"], st["sx"], to_dev_i32(st["or2a"]),
                                       to_dev_i32(st["oo"]), inp["w13"], inp["w13_sf"], act,
                                       act_sf, ws)
            return torch.cat([act.view(-1), act_sf.view(torch.uint8).view(-1)])
        act = torch.empty(wl.R, wl.I, dtype=torch.bfloat16, device=dev())
        C.moe_grouped_gemm1_swiglu(shape, inp["x"], None, to_dev_i32(st["or2a"]),
                                   to_dev_i32(st["oo"]), inp["w13"], None, act, None, ws)
        return act
    y = torch.empty(wl.R, wl.H, dtype=torch.bfloat16, device=dev())
    C.moe_grouped_gemm2(shape, st["a_in"], st["sa_in"], to_dev_i32(st["oo"]), inp["w2"],
                        inp.get("w2_sf"), y, ws)
    return y


@pytest.mark.parametrize("which", ["gemm1", "gemm2"])
@pytest.mark.parametrize("case", list(CASES))
def test_injected_stall_reports_timeout_and_context_survives(case, which):
    wl = CASES[case]
    st = _setup(wl)
    clean = _run(wl, st, which).clone()
    torch.cuda.synchronize()
    assert C.moe_get_device_status(st["ws"]) == 0
    limit_s = 0.05
    C.moe_debug_set_wait_limit_ns(int(limit_s * 1e9))
    C.moe_debug_inject_stall(True)
    try:
        t0 = time.perf_counter()
        _run(wl, st, which)
        torch.cuda.synchronize()
        elapsed = time.perf_counter() - t0
        assert C.moe_get_device_status(st["ws"]) == C.MOE_ERR_DEVICE_TIMEOUT
        # every role (in SM pairs, both CTAs) unwinds within a few limits, not one per wait
        assert elapsed < 10 * limit_s, f"stalled launch took {elapsed:.3f} s"
    finally:
        C.moe_debug_inject_stall(False)
        C.moe_debug_set_wait_limit_ns(0)
    again = _run(wl, st, which)
    torch.cuda.synchronize()
    assert C.moe_get_device_status(st["ws"]) == 0
    assert torch.equal(again.view(torch.uint8), clean.view(torch.uint8)), "results changed"
    if case == "bf16_swap":   # and the clean result is the oracle's
        inp, oo, or2a = st["inp"], st["oo"], st["or2a"]
        ex = np.repeat(np.arange(wl.E_all), np.diff(oo)).astype(np.int32)
        if which == "gemm1":
            ref = oracle.gemm1_bf16_rows(I.bits(inp["x"]), I.bits(inp["w13"]), or2a // wl.k, ex)
        else:
            ref = oracle.gemm2_bf16_rows(I.bits(st["a_in"]), I.bits(inp["w2"]),
                                         np.arange(wl.R), ex)
        assert_close(f64(again), ref, what=f"{which} after recovery")


def test_front_end_barrier_timeout_and_recovery():
    """moe_forward's large-batch front end (routing and permutation in one cooperative
    launch) waits at a grid-wide barrier; with the hook it waits for one CTA too many, the
    bounded wait expires, the status reads MOE_ERR_DEVICE_TIMEOUT (reading it resets the
    barrier's words), and the next call gives the clean call's bits again."""
    wl = I.Workload("fe", 300, 256, 128, 16, 4)
    inp = I.make_inputs(wl, 0, dev())
    shape = C.MoeShape.from_workload(wl)
    ws = workspace(shape)

    def fwd():
        out = torch.empty(wl.T, wl.H, dtype=torch.bfloat16, device=dev())
        C.moe_forward(shape, inp["x"], inp["logits"], inp["w13"], None, inp["w2"], None, out,
                      None, ws)
        torch.cuda.synchronize()
        return out

    clean = fwd()
    assert C.moe_get_device_status(ws) == 0
    C.moe_debug_set_wait_limit_ns(50_000_000)
    C.moe_debug_inject_stall(True)
    try:
        fwd()
        assert C.moe_get_device_status(ws) == C.MOE_ERR_DEVICE_TIMEOUT
    finally:
        C.moe_debug_inject_stall(False)
        C.moe_debug_set_wait_limit_ns(0)
    again = fwd()
    assert C.moe_get_device_status(ws) == 0
    assert torch.equal(again.view(torch.int16), clean.view(torch.int16))
