"""Failure detection without a GPU fault: a test hook leaves one pipeline stage of a
grouped-GEMM launch unfilled, the consumer's bounded mbarrier wait (shortened to 50 ms)
expires, every role of the kernel unwinds, the status word reads MOE_ERR_DEVICE_TIMEOUT,
and the context stays usable: the next launches give correct results."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import assert_close, dev, f64, oracle_route, to_dev_i32, workspace
from mixture_experts_routed_histogram_b200 import _capi as C
from mixture_experts_routed_histogram_b200 import inputs as I

pytestmark = pytest.mark.gpu


def _case():
    wl = I.WORKLOADS["tiny"]
    inp = I.make_inputs(wl, 0, dev())
    oids, _ = oracle_route(wl, inp["logits"])
    _, oo, or2a, _ = oracle.permute(oids, wl.E)
    return wl, inp, oo, or2a


def _gemm1(shape, wl, inp, oo, or2a, ws):
    act = torch.empty(wl.R, wl.I, dtype=torch.bfloat16, device=dev())
    C.moe_grouped_gemm1_swiglu(shape, inp["x"], None, to_dev_i32(or2a), to_dev_i32(oo),
                               inp["w13"], None, act, None, ws)
    return act


def _gemm2(shape, wl, inp, oo, act, ws):
    y = torch.empty(wl.R, wl.H, dtype=torch.bfloat16, device=dev())
    C.moe_grouped_gemm2(shape, act, None, to_dev_i32(oo), inp["w2"], None, y, ws)
    return y


@pytest.mark.parametrize("which", ["gemm1", "gemm2"])
def test_injected_stall_reports_timeout_and_context_survives(which):
    wl, inp, oo, or2a = _case()
    shape = C.MoeShape.from_workload(wl)
    ws = workspace(shape)
    g = torch.Generator(device=dev()).manual_seed(3)
    act_in = torch.randn(wl.R, wl.I, generator=g, device=dev()).to(torch.bfloat16)
    C.moe_debug_set_wait_limit_ns(50_000_000)
    C.moe_debug_inject_stall(True)
    try:
        if which == "gemm1":
            _gemm1(shape, wl, inp, oo, or2a, ws)
        else:
            _gemm2(shape, wl, inp, oo, act_in, ws)
        torch.cuda.synchronize()
        assert C.moe_get_device_status(ws) == C.MOE_ERR_DEVICE_TIMEOUT
    finally:
        C.moe_debug_inject_stall(False)
        C.moe_debug_set_wait_limit_ns(0)
    # the same launch again, without the hook: correct, and no status
    ex = np.repeat(np.arange(wl.E), np.diff(oo)).astype(np.int32)
    if which == "gemm1":
        out = _gemm1(shape, wl, inp, oo, or2a, ws)
        ref = oracle.gemm1_bf16_rows(I.bits(inp["x"]), I.bits(inp["w13"]), or2a // wl.k, ex)
    else:
        out = _gemm2(shape, wl, inp, oo, act_in, ws)
        ref = oracle.gemm2_bf16_rows(I.bits(act_in), I.bits(inp["w2"]), np.arange(wl.R), ex)
    torch.cuda.synchronize()
    assert C.moe_get_device_status(ws) == 0
    assert_close(f64(out), ref, what=f"{which} after recovery")
