"""Host-side checks of the C ABI that need no GPU: the library loads, exports every
function include/moe.h declares, and rejects bad arguments before launching anything."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            with open(os.path.join(ROOT, "include", fn)) as f:
                names |= set(re.findall(r"^MOE_API[^(]*?\b(moe_\w+)\(", f.read(), re.M))
    return names


def test_header_declares_the_boundary():
    need = {"moe_route", "moe_permute", "moe_grouped_gemm1_swiglu", "moe_grouped_gemm2",
            "moe_combine", "moe_forward", "moe_workspace_size", "moe_quantize_x"}
    assert need <= _declared()


def test_library_exports_every_declared_symbol(moelib):
    lib = ctypes.CDLL(moelib.lib_path())
    missing = [n for n in sorted(_declared()) if not hasattr(lib, n)]
    assert not missing, missing
    assert set(moelib.EXPORTS) == _declared()


def _shape(moelib, **kw):
    base = dict(T=64, H=256, I=128, E=8, k=2, score="softmax", renorm=True, dtype="bf16")
    base.update(kw)
    return moelib.MoeShape.of(**base)


@pytest.mark.parametrize("kw,status", [
    (dict(k=0), 1), (dict(k=9), 1), (dict(T=-1), 1), (dict(H=0), 1),
    (dict(E=2000, k=2), 2), (dict(k=33, E=64), 2), (dict(H=100), 2), (dict(I=96), 2),
    (dict(dtype="fp8_mxfp4", H=192), 2), (dict(T=2 ** 29, k=8), 2),
    # ReLU2 is BF16 only; shared experts count against the slot and expert limits
    (dict(dtype="fp8_mxfp4", act="relu2"), 2), (dict(n_shared=-1), 1),
    (dict(k=30, E=64, n_shared=3), 2), (dict(E=1023, n_shared=2), 2),
])
def test_shape_validation(moelib, kw, status):
    L = moelib.load()
    s = _shape(moelib, **kw)
    assert L.moe_workspace_size(ctypes.byref(s)) == 0
    assert L.moe_route(ctypes.byref(s), 16, 16, 16, None) == status
    assert L.moe_forward(ctypes.byref(s), 16, 16, 16, None, 16, None, 16, None, 256, 1 << 30,
                         None) == status


def test_unknown_activation_is_rejected(moelib):
    L = moelib.load()
    s = _shape(moelib)
    s.activation = 7
    assert L.moe_workspace_size(ctypes.byref(s)) == 0
    assert L.moe_route(ctypes.byref(s), 16, 16, 16, None) == moelib.MOE_ERR_INVALID_ARG


def test_shared_experts_grow_the_routed_row_space(moelib):
    L = moelib.load()
    a = L.moe_workspace_size(ctypes.byref(_shape(moelib, T=256)))
    b = L.moe_workspace_size(ctypes.byref(_shape(moelib, T=256, n_shared=1)))
    assert b - a >= 256 * (256 + 128) * 2          # one more row of act and y per token


def test_pointer_validation(moelib):
    L = moelib.load()
    s = _shape(moelib)
    assert L.moe_route(ctypes.byref(s), None, 16, 16, None) == moelib.MOE_ERR_INVALID_ARG
    assert L.moe_route(ctypes.byref(s), 18, 16, 16, None) == moelib.MOE_ERR_MISALIGNED
    need = L.moe_workspace_size(ctypes.byref(s))
    assert need > 0
    assert L.moe_forward(ctypes.byref(s), 16, 16, 16, None, 16, None, 16, None, 256, need - 1,
                         None) == moelib.MOE_ERR_WORKSPACE_TOO_SMALL
    assert L.moe_forward(ctypes.byref(s), 16, 16, 16, None, 16, None, 16, None, 272, need,
                         None) == moelib.MOE_ERR_MISALIGNED
    assert L.moe_quantize_weights_mxfp4(4, 48, 16, 16, 16, None) == moelib.MOE_ERR_UNSUPPORTED_SHAPE


def test_zero_tokens_is_a_noop(moelib):
    L = moelib.load()
    s = _shape(moelib, T=0)
    assert L.moe_route(ctypes.byref(s), None, None, None, None) == 0
    assert L.moe_combine(ctypes.byref(s), None, None, None, None, None) == 0


def test_workspace_size_grows_with_tokens(moelib):
    L = moelib.load()
    # (decode-sized T <= 64 also reserves K-split partial sums, so compare larger T)
    a = L.moe_workspace_size(ctypes.byref(_shape(moelib, T=128)))
    b = L.moe_workspace_size(ctypes.byref(_shape(moelib, T=256)))
    R = 128 * 2
    assert b - a >= R * (256 + 128) * 2


def test_status_strings(moelib):
    for st in range(8):
        assert moelib.status_string(st) != "unknown status"


@pytest.mark.parametrize("kw", [dict(T=1), dict(T=64, n_shared=1), dict(T=8192, E=128, k=8),
                                dict(T=300, E=1000, k=32, dtype="fp8_mxfp4")])
def test_workspace_regions_are_disjoint_and_inside(moelib, kw):
    """The routing-metadata regions of the forward's workspace: 256-byte aligned, past the
    status block, inside moe_workspace_size, pairwise disjoint, and of the documented size."""
    s = _shape(moelib, **kw)
    total = moelib.moe_workspace_size(s)
    R, E = s.T * (s.k + s.n_shared), s.E + s.n_shared
    want = {moelib.MOE_WS_IDS: 4 * R, moelib.MOE_WS_W: 4 * R, moelib.MOE_WS_COUNTS: 4 * E,
            moelib.MOE_WS_OFFSETS: 4 * (E + 1), moelib.MOE_WS_ROW2ASSIGN: 4 * R,
            moelib.MOE_WS_ASSIGN2ROW: 4 * R}
    spans = []
    for region, nbytes in want.items():
        off, n = moelib.moe_workspace_region(s, region)
        assert n == nbytes and off % 256 == 0 and off >= 256 and off + n <= total
        spans.append((off, off + n))
    spans.sort()
    assert all(a[1] <= b[0] for a, b in zip(spans, spans[1:]))


def test_workspace_region_rejects_bad_arguments(moelib):
    L = moelib.load()
    s = _shape(moelib)
    off, n = ctypes.c_size_t(), ctypes.c_size_t()
    assert L.moe_workspace_region(ctypes.byref(s), 6, ctypes.byref(off), ctypes.byref(n)) == 1
    assert L.moe_workspace_region(ctypes.byref(s), -1, ctypes.byref(off), ctypes.byref(n)) == 1
    assert L.moe_workspace_region(ctypes.byref(s), 0, None, ctypes.byref(n)) == 1
    bad = _shape(moelib, k=9)
    assert L.moe_workspace_region(ctypes.byref(bad), 0, ctypes.byref(off), ctypes.byref(n)) == 1
