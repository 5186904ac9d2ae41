"""moe_forward captured into a CUDA graph: every launch (programmatic dependent launches,
memsets) is capturable, and replaying the graph gives the same bits as the eager call,
replay after replay, with new inputs copied into the captured buffers between replays."""
import pytest
import torch

from gpu_util import dev, workspace
from mixture_experts_routed_histogram_b200 import _capi as C
from mixture_experts_routed_histogram_b200 import inputs as I

pytestmark = pytest.mark.gpu

CASES = {
    "bf16_many_tiles": I.Workload("g1", 1000, 512, 256, 8, 4),
    "bf16_decode_t8": I.Workload("decode", 8, 512, 256, 8, 2, routing="zipf"),
    "fp8_t300": I.Workload("g3", 300, 256, 256, 4, 2, dtype="fp8_mxfp4"),
}


@pytest.mark.parametrize("name", list(CASES))
def test_forward_graph_replay_matches_eager(name):
    wl = CASES[name]
    shape = C.MoeShape.from_workload(wl)
    ws = workspace(shape)
    a = I.make_inputs(wl, 0, dev())
    b = I.make_inputs(wl, 1, dev())
    x = a["x"].clone()
    logits = a["logits"].clone()
    out = torch.empty(wl.T, wl.H, dtype=torch.bfloat16, device=dev())

    def fwd():
        C.moe_forward(shape, x, logits, a["w13"], a["w13_sf"], a["w2"], a["w2_sf"], out, None, ws)

    # eager results for both input sets (b reuses a's weights)
    fwd()
    torch.cuda.synchronize()
    eager_a = out.clone()
    x.copy_(b["x"])
    logits.copy_(b["logits"])
    fwd()
    torch.cuda.synchronize()
    eager_b = out.clone()
    assert C.moe_get_device_status(ws) == 0

    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            fwd()
    torch.cuda.current_stream().wait_stream(s)
    for src, want in [(a, eager_a), (b, eager_b), (a, eager_a)]:
        x.copy_(src["x"])
        logits.copy_(src["logits"])
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16), want.view(torch.int16))
    assert C.moe_get_device_status(ws) == 0
    del g
