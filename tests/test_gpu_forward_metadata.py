"""The routing metadata moe_forward itself computes -- top-k ids and weights, per-expert
counts, offsets and the expert-sorted permutation (row2assign, assign2row) -- read back
from its workspace (moe_workspace_region) and compared with the oracle's routing and
permutation: bit for bit for the integers, weights to the routing test's fp32 tolerance.

This pins both front ends of the forward pass: the single-CTA routing + permutation kernel
of decode-sized batches (T <= 64, at most 256 experts) and the multi-kernel one of larger
batches, including exact logit ties (the lower expert index wins; within an expert,
rows keep ascending assignment order)."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import dev, oracle_route, workspace
from mixture_experts_routed_histogram_b200 import _capi as C
from mixture_experts_routed_histogram_b200 import inputs as I

pytestmark = pytest.mark.gpu

W = I.WORKLOADS

CASES = {
    # decode-sized front end (one CTA routes and permutes)
    "decode_T1": (W["decode"].with_T(1), False),
    "decode_T8": (W["decode"].with_T(8), False),
    "decode_T32": (W["decode"].with_T(32), False),
    "decode_T64": (W["decode"].with_T(64), False),
    "tiny_ties": (W["tiny"], True),
    "shared1_t40": (I.Workload("sh1", 40, 256, 128, 8, 2, n_shared=1), False),
    "e256_k32_t64_ties": (I.Workload("w256", 64, 256, 128, 256, 32), True),
    "e255_k31_shared1_t17": (I.Workload("w255", 17, 256, 128, 255, 31, n_shared=1), True),
    "sigmoid_top1_t50": (I.Workload("sg", 50, 256, 128, 16, 1, score="sigmoid", renorm=False),
                         False),
    # larger batches (routing, histogram, scan and scatter kernels)
    "decode_T128": (W["decode"].with_T(128), False),
    "ties_e64_k4_t300": (I.Workload("ties", 300, 256, 128, 64, 4), True),
    "e1000_k32_t40": (I.Workload("wide", 40, 256, 128, 1000, 32, routing="uniform"), False),
    "shared2_t500": (I.Workload("sh2", 500, 512, 256, 16, 4, n_shared=2), False),
    "qwen3_30b_a3b": (W["qwen3_30b_a3b"], False),
    # 128-token chunks, three scatter rounds per chunk (block-scaled weights)
    "fp8_mxfp4_T16384": (W["fp8_mxfp4"].with_T(16384), False),
}


def _region(ws, shape, region, dtype):
    off, n = C.moe_workspace_region(shape, region)
    return ws[off:off + n].view(dtype).cpu().numpy()


@pytest.mark.parametrize("name", list(CASES))
def test_forward_metadata_bitexact(name):
    wl, ties = CASES[name]
    inp = I.make_inputs(wl, 0, dev())
    lg = inp["logits"]
    if ties:   # coarse logits: many exact ties between experts
        lg = torch.round(lg * 2) / 2
    shape = C.MoeShape.from_workload(wl)
    ws = workspace(shape)
    out = torch.empty(wl.T, wl.H, dtype=torch.bfloat16, device=dev())
    C.moe_forward(shape, inp["x"], lg, inp["w13"], inp.get("w13_sf"), inp["w2"], inp.get("w2_sf"),
                  out, None, ws)
    torch.cuda.synchronize()
    assert C.moe_get_device_status(ws) == 0
    oids, ow = oracle_route(wl, lg)
    oc, oo, or2a, oa2r = oracle.permute(oids, wl.E_all)
    ks = wl.k + wl.n_shared
    ids = _region(ws, shape, C.MOE_WS_IDS, torch.int32).reshape(wl.T, ks)
    w = _region(ws, shape, C.MOE_WS_W, torch.float32).reshape(wl.T, ks)
    assert np.array_equal(ids, oids)
    assert np.allclose(w, ow, rtol=2e-6, atol=2e-7)
    assert np.array_equal(_region(ws, shape, C.MOE_WS_COUNTS, torch.int32), oc)
    assert np.array_equal(_region(ws, shape, C.MOE_WS_OFFSETS, torch.int32), oo)
    assert np.array_equal(_region(ws, shape, C.MOE_WS_ROW2ASSIGN, torch.int32), or2a)
    assert np.array_equal(_region(ws, shape, C.MOE_WS_ASSIGN2ROW, torch.int32), oa2r)


def test_forward_metadata_with_ids_out():
    """With ids_out given the ids go there; the other regions are filled the same way."""
    wl = W["decode"].with_T(8)
    inp = I.make_inputs(wl, 0, dev())
    shape = C.MoeShape.from_workload(wl)
    ws = workspace(shape)
    out = torch.empty(wl.T, wl.H, dtype=torch.bfloat16, device=dev())
    ids = torch.full((wl.T, wl.k), -1, dtype=torch.int32, device=dev())
    C.moe_forward(shape, inp["x"], inp["logits"], inp["w13"], None, inp["w2"], None, out, ids,
                  ws)
    torch.cuda.synchronize()
    oids, _ = oracle_route(wl, inp["logits"])
    _, _, or2a, oa2r = oracle.permute(oids, wl.E_all)
    assert np.array_equal(ids.cpu().numpy(), oids)
    assert np.array_equal(_region(ws, shape, C.MOE_WS_ROW2ASSIGN, torch.int32), or2a)
    assert np.array_equal(_region(ws, shape, C.MOE_WS_ASSIGN2ROW, torch.int32), oa2r)
