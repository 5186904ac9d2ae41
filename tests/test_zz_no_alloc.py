"""moe_permute_noalloc: the permutation for callers that cannot pass a workspace (for
example host code whose device memory is a fixed pool reserved at start-up, with no
scratch buffer to hand down).  Its scratch is a static device array inside libmoe.so;
its results must equal moe_permute's and the oracle's, bit for bit, call after call.

This file is collected last on purpose: it runs after every other test, and also passes
alone in a fresh process."""
import numpy as np
import pytest
import torch

import oracle
from mixture_experts_routed_histogram_b200 import _capi as C

pytestmark = pytest.mark.gpu


def _ids(T, k, E, seed, n_shared=0):
    """Routed ids [T][k] (one expert skewed) followed by the n_shared shared-expert slots."""
    rng = np.random.default_rng(seed)
    ids = rng.integers(0, E, (T, k)).astype(np.int32)
    ids[rng.random((T, k)) < 0.3] = E // 3
    shared = np.tile(np.arange(E, E + n_shared, dtype=np.int32), (T, 1))
    return np.ascontiguousarray(np.concatenate([ids, shared], axis=1))


def _outputs(E, R):
    dev = torch.device("cuda", 0)
    return (torch.full((E,), -7, dtype=torch.int32, device=dev),
            torch.full((E + 1,), -7, dtype=torch.int32, device=dev),
            torch.full((max(R, 1),), -7, dtype=torch.int32, device=dev),
            torch.full((max(R, 1),), -7, dtype=torch.int32, device=dev))


def _compare_twice(T, k, E, n_shared=0):
    shape = C.MoeShape.of(T, 256, 128, E, k, n_shared=n_shared)
    E_all, R = E + n_shared, T * (k + n_shared)
    ws = torch.empty(C.moe_workspace_size(shape), dtype=torch.uint8, device="cuda")
    C.moe_workspace_init(ws)
    for call, seed in enumerate((1, 2)):          # two calls in a row, different inputs
        ids_h = _ids(T, k, E, seed + 10 * call, n_shared)
        ids = torch.from_numpy(ids_h).cuda()
        ref = _outputs(E_all, R)
        got = _outputs(E_all, R)
        C.moe_permute(shape, ids, *ref, ws)
        C.moe_permute_noalloc(shape, ids, *got)
        torch.cuda.synchronize()
        for r, g in zip(ref, got):
            assert torch.equal(r, g), f"call {call}"
        oc, oo, or2a, oa2r = oracle.permute(ids_h, E_all)
        for g, o in zip(got, (oc, oo, or2a, oa2r)):
            assert np.array_equal(g.cpu().numpy()[:o.size], o), f"call {call} vs oracle"
        assert C.moe_get_device_status(ws) == 0


@pytest.mark.parametrize("T,k,E", [(4096, 8, 128), (300, 10, 512),
                                   # the documented limit: (2 * 128 + 1) * 510 <= 131072 ints
                                   (16384, 2, 510)])
def test_noalloc_permute_matches_workspace_permute_and_oracle_twice(T, k, E):
    _compare_twice(T, k, E)


def test_noalloc_permute_with_a_shared_expert_at_the_limit():
    """E + n_shared = 510 experts in the permutation: still inside the static scratch."""
    _compare_twice(16384, 2, 509, n_shared=1)


def test_noalloc_permute_zero_tokens():
    shape = C.MoeShape.of(0, 256, 128, 8, 2)
    counts, offsets, r2a, a2r = _outputs(8, 0)
    C.moe_permute_noalloc(shape, None, counts, offsets, r2a, a2r)
    torch.cuda.synchronize()
    assert int(counts.abs().sum()) == 0 and int(offsets.abs().sum()) == 0


@pytest.mark.parametrize("T,E,k,n_shared", [(60000, 1024, 10, 0),   # far beyond the scratch
                                            (16384, 511, 2, 0),     # (257 * 511) > 131072
                                            (16384, 510, 2, 1)])    # 511 with the shared one
def test_noalloc_permute_rejects_sizes_beyond_its_scratch(T, E, k, n_shared):
    shape = C.MoeShape.of(T, 256, 128, E, k, n_shared=n_shared)
    E_all, R = E + n_shared, T * (k + n_shared)
    with pytest.raises(C.MoeError) as ex:
        C.moe_permute_noalloc(shape, torch.zeros(R, dtype=torch.int32, device="cuda"),
                              *_outputs(E_all, R))
    assert ex.value.status == C.MOE_ERR_UNSUPPORTED_SHAPE
