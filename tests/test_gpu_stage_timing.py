"""moe_debug_time_stages: the events moe_forward records name every stage of the path the
shape takes (the front end -- routing and permutation in one launch at every batch size;
FP8 quantisation; K-split decode GEMMs), each stage takes positive time, the output is the same bits as an untimed
forward, and turning it off stops the recording."""
import pytest
import torch

from gpu_util import dev, workspace
from mixture_experts_routed_histogram_b200 import _capi as C
from mixture_experts_routed_histogram_b200 import inputs as I

pytestmark = pytest.mark.gpu

CASES = {
    "small_batch": (I.WORKLOADS["tiny"], ["route_permute", "gemm1_swiglu", "gemm2", "combine"]),
    "ksplit_decode": (I.Workload("ks", 24, 512, 3072, 4, 2, routing="zipf"),
                      ["route_permute", "gemm1_swiglu", "gemm2", "combine"]),
    "bf16_many_tiles": (I.Workload("m", 1000, 512, 256, 8, 4),
                        ["route_permute", "gemm1_swiglu", "gemm2", "combine"]),
    "fp8": (I.Workload("f8", 300, 256, 256, 4, 2, dtype="fp8_mxfp4"),
            ["route_permute", "quantize_x", "gemm1_swiglu", "gemm2", "combine"]),
}


@pytest.mark.parametrize("name", list(CASES))
def test_forward_stage_events(name):
    wl, stages = CASES[name]
    shape = C.MoeShape.from_workload(wl)
    ws = workspace(shape)
    inp = I.make_inputs(wl, 0, dev())
    out = torch.empty(wl.T, wl.H, dtype=torch.bfloat16, device=dev())

    def fwd():
        C.moe_forward(shape, inp["x"], inp["logits"], inp["w13"], inp["w13_sf"], inp["w2"],
                      inp["w2_sf"], out, None, ws)

    fwd()
    torch.cuda.synchronize()
    ref = out.clone()
    assert C.moe_debug_stage_times() == []
    C.moe_debug_time_stages(True)
    try:
        out.zero_()
        fwd()
        got = C.moe_debug_stage_times()
    finally:
        C.moe_debug_time_stages(False)
    assert [n for n, _ in got] == stages
    assert all(t > 0.0 for _, t in got)
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
    fwd()
    assert C.moe_debug_stage_times() == []
    assert C.moe_get_device_status(ws) == 0
