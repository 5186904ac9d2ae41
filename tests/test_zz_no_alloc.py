"""moe_permute_noalloc: the permutation for callers that cannot pass a workspace (for
example host code whose device memory is a fixed pool reserved at start-up, with no
scratch buffer to hand down).  Its scratch is a static device array inside libmoe.so;
its results must equal moe_permute's, bit for bit, call after call.

This file is collected last on purpose: it runs after every other test, and also passes
alone in a fresh process."""
import numpy as np
import pytest
import torch

from mixture_experts_routed_histogram_b200 import _capi as C

pytestmark = pytest.mark.gpu


def _ids(T, k, E, seed):
    rng = np.random.default_rng(seed)
    ids = rng.integers(0, E, (T, k)).astype(np.int32)
    ids[rng.random((T, k)) < 0.3] = E // 3          # skew one expert
    return torch.from_numpy(ids).cuda()


def _outputs(E, R):
    dev = torch.device("cuda", 0)
    return (torch.full((E,), -7, dtype=torch.int32, device=dev),
            torch.full((E + 1,), -7, dtype=torch.int32, device=dev),
            torch.full((max(R, 1),), -7, dtype=torch.int32, device=dev),
            torch.full((max(R, 1),), -7, dtype=torch.int32, device=dev))


@pytest.mark.parametrize("T,k,E", [(4096, 8, 128), (300, 10, 512)])
def test_noalloc_permute_matches_workspace_permute_twice(T, k, E):
    shape = C.MoeShape.of(T, 256, 128, E, k)
    ws = torch.empty(C.moe_workspace_size(shape), dtype=torch.uint8, device="cuda")
    C.moe_workspace_init(ws)
    for call, seed in enumerate((1, 2)):          # two calls in a row, different inputs
        ids = _ids(T, k, E, seed + 10 * call)
        ref = _outputs(E, T * k)
        got = _outputs(E, T * k)
        C.moe_permute(shape, ids, *ref, ws)
        C.moe_permute_noalloc(shape, ids, *got)
        torch.cuda.synchronize()
        for r, g in zip(ref, got):
            assert torch.equal(r, g), f"call {call}"
        assert C.moe_get_device_status(ws) == 0


def test_noalloc_permute_rejects_sizes_beyond_its_scratch():
    shape = C.MoeShape.of(60000, 256, 128, 1024, 10)   # (2 * 128 + 1) * 1024 ints > 131072
    E, R = 1024, 600000
    with pytest.raises(C.MoeError) as ex:
        C.moe_permute_noalloc(shape, torch.zeros(R, dtype=torch.int32, device="cuda"),
                              *_outputs(E, R))
    assert ex.value.status == C.MOE_ERR_UNSUPPORTED_SHAPE
