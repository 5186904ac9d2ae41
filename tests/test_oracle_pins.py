"""Pins for the fp64 CPU oracle: every oracle function is checked here against something
other than itself -- the published format tables, library number-format casts, closed
forms, brute force on tiny inputs, invariants, and the block-scaled -> BF16 reduction.

A plausible slip anywhere in the oracle (a dropped term, a wrong sign or index, a
transposed operand, a wrong tie rule) fails at least one test below.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
from scipy.special import expit, softmax

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _json(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def _bf16_bits(a: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _bits_to_f64(b: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()


def _torch_e4m3(v) -> np.ndarray:
    """Library e4m3 cast (round to nearest even; NaN beyond the format's range)."""
    return torch.tensor(np.asarray(v, np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def _silu(g):
    return g * expit(g)


# ------------------------------------------------------------------ number formats

def test_e4m3_decode_all_codes_match_library(orc):
    codes = np.arange(256, dtype=np.uint8)
    ours = orc.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    fin = ~np.isnan(ref)
    assert np.array_equal(ours[fin], ref[fin])
    assert np.array_equal(np.signbit(ours[fin]), np.signbit(ref[fin]))


def test_e4m3_named_values_and_nan(orc):
    g = _json("formats.json")
    for code, val in g["e4m3_named_values"].items():
        v = orc.e4m3_decode([int(code, 16)])[0]
        assert v == val and np.signbit(v) == np.signbit(val), code
    for code in g["e4m3_nan_codes"]:
        assert np.isnan(orc.e4m3_decode([int(code, 16)])[0])


def test_e4m3_encode_matches_library_rne(orc):
    rng = np.random.default_rng(1)
    mags = np.exp(rng.uniform(np.log(1e-4), np.log(448.0), 4000)).astype(np.float32)
    vals = mags * rng.choice([-1.0, 1.0], mags.size).astype(np.float32)
    # every exact midpoint between neighbouring finite codes is a tie
    pos = orc.e4m3_decode(np.arange(0, 0x7f, dtype=np.uint8))
    mids = ((pos[:-1] + pos[1:]) / 2).astype(np.float32)
    vals = np.concatenate([vals, mids, -mids, [0.0, -0.0]]).astype(np.float32)
    assert np.array_equal(orc.e4m3_encode(vals), _torch_e4m3(vals))


def test_e4m3_saturates(orc):
    for v, want in _json("formats.json")["e4m3_satfinite_cases"]:
        assert orc.e4m3_decode(orc.e4m3_encode([v]))[0] == want


def test_e4m3_round_trip(orc):
    codes = np.array([c for c in range(256) if c not in (0x7f, 0xff)], np.uint8)
    assert np.array_equal(orc.e4m3_encode(orc.e4m3_decode(codes)), codes)


def test_e2m1_table_matches_spec(orc):
    want = np.array(_json("formats.json")["e2m1_values_by_code"])
    got = orc.e2m1_decode(np.arange(16, dtype=np.uint8))
    assert np.array_equal(got, want) and np.array_equal(np.signbit(got), np.signbit(want))


def test_e2m1_rne_ties_by_hand(orc):
    for v, want in _json("formats.json")["e2m1_rne_cases"]:
        assert orc.e2m1_decode(orc.e2m1_encode([v]))[0] == want, v


def test_e2m1_encode_is_nearest_with_even_ties(orc):
    """Brute force: the encoded value is a nearest grid point; on a tie it has an even
    mantissa bit; beyond 6 it saturates to 6."""
    grid = orc.e2m1_decode(np.arange(8, dtype=np.uint8))  # 0 .. 6
    rng = np.random.default_rng(2)
    vals = np.concatenate([rng.uniform(-8, 8, 3000), (grid[:-1] + grid[1:]) / 2])
    codes = orc.e2m1_encode(vals)
    for v, c in zip(vals, codes):
        a = min(abs(v), 6.0)
        d = np.abs(grid - a)
        best = np.flatnonzero(d == d.min())
        mag = int(c) & 7
        assert mag in best
        if len(best) == 2:
            assert mag % 2 == 0
        assert ((int(c) >> 3) & 1) == (1 if np.signbit(v) else 0)


def test_e2m1_round_trip(orc):
    codes = np.arange(16, dtype=np.uint8)
    assert np.array_equal(orc.e2m1_encode(orc.e2m1_decode(codes)), codes)


def test_ue8m0_matches_library(orc):
    b = np.arange(256, dtype=np.uint8)
    ours = orc.ue8m0_decode(b)
    ref = torch.from_numpy(b).view(torch.float8_e8m0fnu).to(torch.float64).numpy()
    assert np.isnan(ours[255]) and np.isnan(ref[255])
    assert np.array_equal(ours[:255], ref[:255])
    for code, val in _json("formats.json")["ue8m0_named_values"].items():
        assert orc.ue8m0_decode([int(code, 16)])[0] == val


def test_bf16_conversions_match_library(orc):
    rng = np.random.default_rng(3)
    v = np.concatenate([rng.standard_normal(3000) * 10.0 ** rng.integers(-30, 30, 3000),
                        [0.0, -0.0, 1.0, -2.5, 3.0e38]]).astype(np.float32)
    ref = torch.tensor(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(orc.f64_to_bf16(v.astype(np.float64)), ref)
    assert np.array_equal(orc.bf16_to_f64(ref), _bits_to_f64(ref))


# ------------------------------------------------------------------ routing

@pytest.mark.parametrize("case", _json("route_example.json")["cases"])
def test_route_hand_examples(orc, case):
    score = orc.SOFTMAX if case["score"] == "softmax" else orc.SIGMOID
    ids, w = orc.route(np.array(case["logits"], np.float32), case["k"], score, case["renorm"])
    assert ids.tolist() == case["ids"]
    assert np.allclose(w, case["w"], rtol=0, atol=1e-15)


def _topk_by_sort(lg, k):
    # np.lexsort: last key is primary -> sort by (-logit, expert index)
    T, E = lg.shape
    out = np.empty((T, k), np.int64)
    for t in range(T):
        order = np.lexsort((np.arange(E), -lg[t].astype(np.float64)))
        out[t] = order[:k]
    return out


@pytest.mark.parametrize("E,k", [(8, 2), (16, 1), (64, 8), (512, 10), (5, 5)])
def test_route_matches_sort_and_closed_form(orc, E, k):
    rng = np.random.default_rng(E * 31 + k)
    lg = rng.standard_normal((40, E)).astype(np.float32)
    lg[3, :] = 0.25                        # an all-tie row
    lg[5, [1, 4 % E]] = lg[5].max() + 1    # a tie at the top
    ids, w = orc.route(lg, k, orc.SOFTMAX, True)
    assert np.array_equal(ids, _topk_by_sort(lg, k))
    # softmax over all E, then renormalise over the selected k (closed form)
    p = softmax(lg.astype(np.float64), axis=1)
    sel = np.take_along_axis(p, ids, axis=1)
    assert np.allclose(w, sel / sel.sum(1, keepdims=True), rtol=1e-13, atol=0)
    assert np.allclose(w.sum(1), 1.0, rtol=0, atol=1e-15)
    # without renormalisation: plain softmax probabilities of the selected experts
    _, w2 = orc.route(lg, k, orc.SOFTMAX, False)
    assert np.allclose(w2, sel, rtol=1e-13, atol=0)
    # sigmoid of the selected logit
    _, ws = orc.route(lg, k, orc.SIGMOID, False)
    assert np.allclose(ws, expit(np.take_along_axis(lg, ids, 1).astype(np.float64)), rtol=1e-14)


def test_route_token_permutation_equivariance(orc):
    rng = np.random.default_rng(7)
    lg = rng.standard_normal((50, 32)).astype(np.float32)
    perm = rng.permutation(50)
    ids, w = orc.route(lg, 4)
    ids_p, w_p = orc.route(lg[perm], 4)
    assert np.array_equal(ids_p, ids[perm]) and np.array_equal(w_p, w[perm])


# ------------------------------------------------------------------ histogram / permutation

@pytest.mark.parametrize("T,E,k,skew", [(64, 8, 2, False), (1000, 128, 8, False),
                                        (257, 16, 1, True), (3, 512, 10, False), (0, 4, 2, False)])
def test_permute_invariants_and_brute_force(orc, T, E, k, skew):
    rng = np.random.default_rng(T + E + k)
    if T:
        if skew:
            lg = rng.standard_normal((T, E)).astype(np.float32)
            lg[:, 3] += 100.0            # every token picks expert 3 first
        else:
            lg = rng.standard_normal((T, E)).astype(np.float32)
        ids, _ = orc.route(lg, k)
    else:
        ids = np.zeros((0, k), np.int32)
    counts, offsets, r2a, a2r = orc.permute(ids, E)
    R = T * k
    flat = ids.reshape(-1)
    assert counts.sum() == R
    assert np.array_equal(counts, np.bincount(flat, minlength=E))
    assert offsets[0] == 0 and np.array_equal(np.diff(offsets), counts)
    assert np.array_equal(np.sort(r2a), np.arange(R))            # bijection
    assert np.array_equal(a2r[r2a], np.arange(R))                # inverse
    # brute force: the stable argsort of the expert ids is exactly row2assign
    assert np.array_equal(r2a, np.argsort(flat, kind="stable"))
    for e in range(E):
        seg = r2a[offsets[e]:offsets[e + 1]]
        assert np.all(flat[seg] == e) and np.all(np.diff(seg) > 0)


def test_permute_rejects_bad_ids(orc):
    with pytest.raises(ValueError):
        orc.permute(np.array([[0, 9]], np.int32), 4)


# ------------------------------------------------------------------ quantisers

def test_quant_fp8_hand_groups(orc):
    """Worked by hand from the 1x128 power-of-two rule: amax 448 -> scale 1; amax 449 ->
    scale 2 (449/2 = 224.5 rounds to 224 on the e4m3 grid, spacing 16 there); amax 1 ->
    scale 2^-8 (1/448 lies in (2^-9, 2^-8]); all zero -> scale 1, codes 0."""
    v = np.zeros((4, 128))
    v[0, 5] = 448.0
    v[1, 0] = 449.0
    v[2, 7] = -1.0
    codes, sc = orc.quant_fp8(v)
    assert sc[:, 0].tolist() == [1.0, 2.0, 2.0 ** -8, 1.0]
    assert orc.e4m3_decode(codes[0, 5:6])[0] == 448.0
    assert orc.e4m3_decode(codes[1, 0:1])[0] == 224.0
    assert orc.e4m3_decode(codes[2, 7:8])[0] == -256.0
    assert not codes[3].any()


def test_quant_fp8_matches_log2_rule_and_library_cast(orc):
    rng = np.random.default_rng(11)
    x = (rng.standard_normal((64, 512)) * 10.0 ** rng.integers(-3, 4, (64, 1))).astype(np.float32)
    xb = _bf16_bits(x)
    xv = _bits_to_f64(xb)
    codes, sc = orc.quant_fp8_bf16(xb)
    for r in range(64):
        for g in range(4):
            grp = xv[r, g * 128:(g + 1) * 128]
            amax = np.abs(grp).max()
            assert sc[r, g] == 2.0 ** math.ceil(math.log2(amax / 448.0))
            assert np.array_equal(codes[r, g * 128:(g + 1) * 128], _torch_e4m3(grp / sc[r, g]))


def test_quant_mxfp4_hand_block(orc):
    """amax 5 -> floor(log2 5) - 2 = 0 -> byte 127; 1 -> 1, 0.75 -> 1 (tie to even),
    0.25 -> 0, -5 -> -4; element 0 sits in the low nibble."""
    w = np.zeros((1, 32), np.float32)
    w[0, :4] = [1.0, 0.75, 0.25, -5.0]
    packed, sf = orc.quant_mxfp4(_bf16_bits(w))
    assert sf.tolist() == [[127]]
    assert packed[0, 0] == (0x2 | (0x2 << 4))        # codes 2 (1.0) and 2 (1.0)
    assert packed[0, 1] == (0x0 | (0xE << 4))        # codes 0 (0.0) and 14 (-4.0)
    z, zsf = orc.quant_mxfp4(np.zeros((1, 32), np.uint16))
    assert zsf.tolist() == [[0]] and not z.any()


def test_quant_mxfp4_matches_spec_rule_and_error_bound(orc):
    rng = np.random.default_rng(12)
    w = (rng.standard_normal((24, 256)) / 16.0).astype(np.float32)
    wb = _bf16_bits(w)
    wv = _bits_to_f64(wb)
    packed, sf = orc.quant_mxfp4(wb)
    deq = orc.mxfp4_dequant(packed, sf)
    for r in range(24):
        for g in range(8):
            blk = wv[r, g * 32:(g + 1) * 32]
            X = math.floor(math.log2(np.abs(blk).max())) - 2
            assert sf[r, g] == X + 127
            # each element is a nearest e2m1 multiple of 2^X (saturating at 6 * 2^X)
            grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6]) * 2.0 ** X
            got = np.abs(deq[r, g * 32:(g + 1) * 32])
            for a, q in zip(np.minimum(np.abs(blk), grid[-1]), got):
                assert abs(a - q) <= np.abs(grid - a).min() + 1e-300
            assert np.all(np.sign(deq[r, g * 32:(g + 1) * 32]) * np.sign(blk) >= 0)


# ------------------------------------------------------------------ expert MLP

def _rand_bf16(rng, shape, scale=1.0):
    return _bf16_bits(rng.standard_normal(shape) * scale)


def _dense_moe_np(xv, lg, k, w13v, w2v, score="softmax", renorm=True):
    """Every expert on every token, then top-k selection by sort and weighting."""
    E = w13v.shape[0]
    I = w13v.shape[1] // 2
    Y = np.stack([(_silu(xv @ w13v[e, :I].T) * (xv @ w13v[e, I:].T)) @ w2v[e].T for e in range(E)])
    ids = _topk_by_sort(lg, k)
    sel = np.take_along_axis(lg.astype(np.float64), ids, 1)
    if score == "softmax":
        w = softmax(sel, axis=1) if renorm else np.take_along_axis(softmax(lg.astype(np.float64), 1), ids, 1)
    else:
        w = expit(sel)
    out = np.zeros_like(xv)
    for t in range(xv.shape[0]):
        for j in range(k):
            out[t] += w[t, j] * Y[ids[t, j], t]
    return out


def test_single_expert_top1_is_dense_swiglu_mlp(orc):
    rng = np.random.default_rng(20)
    T, H, I = 9, 64, 48
    xb = _rand_bf16(rng, (T, H))
    w13 = _rand_bf16(rng, (1, 2 * I, H), H ** -0.5)
    w2 = _rand_bf16(rng, (1, H, I), I ** -0.5)
    lg = rng.standard_normal((T, 1)).astype(np.float32)
    ids, w = orc.route(lg, 1)
    assert np.all(ids == 0) and np.all(w == 1.0)
    out, outb = orc.forward_bf16(xb, ids, w, w13, w2)
    xv, g13, g2 = _bits_to_f64(xb), _bits_to_f64(w13)[0], _bits_to_f64(w2)[0]
    dense = (_silu(xv @ g13[:I].T) * (xv @ g13[I:].T)) @ g2.T
    assert np.allclose(out, dense, rtol=1e-12, atol=1e-14)
    assert np.array_equal(outb, orc.f64_to_bf16(out))


@pytest.mark.parametrize("T,E,k,score", [(8, 6, 2, "softmax"), (5, 4, 4, "softmax"),
                                         (7, 6, 1, "sigmoid"), (1, 3, 2, "softmax")])
def test_forward_bf16_brute_force_tiny(orc, T, E, k, score):
    rng = np.random.default_rng(T * 100 + E * 10 + k)
    H = I = 32
    xb = _rand_bf16(rng, (T, H))
    w13 = _rand_bf16(rng, (E, 2 * I, H), H ** -0.5)
    w2 = _rand_bf16(rng, (E, H, I), I ** -0.5)
    lg = rng.standard_normal((T, E)).astype(np.float32)
    sc = orc.SOFTMAX if score == "softmax" else orc.SIGMOID
    ids, w = orc.route(lg, k, sc, score == "softmax")
    out, _ = orc.forward_bf16(xb, ids, w, w13, w2)
    ref = _dense_moe_np(_bits_to_f64(xb), lg, k, _bits_to_f64(w13), _bits_to_f64(w2), score,
                        score == "softmax")
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-13)


# ReLU2 variant (FlashInfer PR #5129, the Nemotron-3.5-Lightning shape): non-gated,
# W1 [E, I, H], act = max(x.W1^T, 0)^2.

def _relu2(g):
    return np.where(g > 0, g * g, 0.0)


def test_single_expert_top1_relu2_is_dense_squared_relu_mlp(orc):
    rng = np.random.default_rng(22)
    T, H, I = 9, 64, 48
    xb = _rand_bf16(rng, (T, H))
    w1 = _rand_bf16(rng, (1, I, H), H ** -0.5)
    w2 = _rand_bf16(rng, (1, H, I), I ** -0.5)
    ids = np.zeros((T, 1), np.int32)
    w = np.ones((T, 1))
    out, _ = orc.forward_bf16(xb, ids, w, w1, w2, act="relu2")
    xv, g1, g2 = _bits_to_f64(xb), _bits_to_f64(w1)[0], _bits_to_f64(w2)[0]
    dense = _relu2(xv @ g1.T) @ g2.T
    assert np.allclose(out, dense, rtol=1e-12, atol=1e-14)


def test_relu2_hand_worked_rows(orc):
    """h = (1, 2, -1, 0.5); rows of W1 chosen so that g = 3.5, -2, 0, 0.25 exactly:
    act = 12.25, 0, 0, 0.0625; with W2 = ones, y = 12.3125 in every column."""
    H, I = 4, 4
    x = np.array([[1.0, 2.0, -1.0, 0.5]])
    w1 = np.array([[[1, 1, 0, 1], [0, -1, 0, 0], [1, 0, 1, 0], [0, 0, 0, 0.5]]], float)
    w2 = np.ones((1, H, I))
    act = orc.gemm1_bf16_rows(_bf16_bits(x), _bf16_bits(w1), np.array([0]), np.array([0]),
                              act="relu2")
    assert np.array_equal(act[0], [12.25, 0.0, 0.0, 0.0625])
    out, _ = orc.forward_bf16(_bf16_bits(x), np.zeros((1, 1), np.int32), np.ones((1, 1)),
                              _bf16_bits(w1), _bf16_bits(w2), act="relu2")
    assert np.array_equal(out[0], np.full(H, 12.3125))


@pytest.mark.parametrize("T,E,k", [(8, 6, 2), (5, 4, 4), (3, 5, 1)])
def test_forward_relu2_brute_force_tiny(orc, T, E, k):
    rng = np.random.default_rng(T * 100 + E * 10 + k + 7)
    H = I = 32
    xb = _rand_bf16(rng, (T, H))
    w1 = _rand_bf16(rng, (E, I, H), H ** -0.5)
    w2 = _rand_bf16(rng, (E, H, I), I ** -0.5)
    lg = rng.standard_normal((T, E)).astype(np.float32)
    ids, w = orc.route(lg, k)
    out, _ = orc.forward_bf16(xb, ids, w, w1, w2, act="relu2")
    xv, g1, g2 = _bits_to_f64(xb), _bits_to_f64(w1), _bits_to_f64(w2)
    Y = np.stack([_relu2(xv @ g1[e].T) @ g2[e].T for e in range(E)])
    sel = _topk_by_sort(lg, k)
    ww = softmax(np.take_along_axis(lg.astype(np.float64), sel, 1), axis=1)
    ref = np.zeros_like(xv)
    for t in range(T):
        for j in range(k):
            ref[t] += ww[t, j] * Y[sel[t, j], t]
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-13)


def test_shared_experts_add_a_dense_mlp_to_the_routed_output(orc):
    """Shared experts: the routed forward plus, for every token, each shared expert's
    dense SwiGLU MLP with weight 1 (an independent numpy formulation)."""
    rng = np.random.default_rng(23)
    T, H, I, E, k, ns = 7, 64, 32, 5, 2, 2
    xb = _rand_bf16(rng, (T, H))
    w13 = _rand_bf16(rng, (E + ns, 2 * I, H), H ** -0.5)
    w2 = _rand_bf16(rng, (E + ns, H, I), I ** -0.5)
    lg = rng.standard_normal((T, E)).astype(np.float32)
    ids, w = orc.route(lg, k, n_shared=ns)
    assert ids.shape == (T, k + ns)
    assert np.array_equal(ids[:, k:], np.tile(np.arange(E, E + ns), (T, 1)))
    assert np.array_equal(w[:, k:], np.ones((T, ns)))
    rid, rw = orc.route(lg, k)
    assert np.array_equal(ids[:, :k], rid) and np.array_equal(w[:, :k], rw)
    out, _ = orc.forward_bf16(xb, ids, w, w13, w2)
    xv, g13, g2 = _bits_to_f64(xb), _bits_to_f64(w13), _bits_to_f64(w2)
    ref = _dense_moe_np(xv, lg, k, g13[:E], g2[:E])
    for s_ in range(ns):
        e = E + s_
        ref += (_silu(xv @ g13[e, :I].T) * (xv @ g13[e, I:].T)) @ g2[e].T
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-13)


def test_forward_token_subset_and_order_equivariance(orc):
    rng = np.random.default_rng(21)
    T, H, I, E, k = 12, 32, 32, 5, 2
    xb = _rand_bf16(rng, (T, H))
    w13 = _rand_bf16(rng, (E, 2 * I, H), H ** -0.5)
    w2 = _rand_bf16(rng, (E, H, I), I ** -0.5)
    lg = rng.standard_normal((T, E)).astype(np.float32)
    ids, w = orc.route(lg, k)
    out, _ = orc.forward_bf16(xb, ids, w, w13, w2)
    sub, _ = orc.forward_bf16(xb, ids, w, w13, w2, tokens=[11, 0, 4])
    assert np.array_equal(sub, out[[11, 0, 4]])
    perm = rng.permutation(T)
    ids_p, w_p = orc.route(lg[perm], k)
    out_p, _ = orc.forward_bf16(xb[perm], ids_p, w_p, w13, w2)
    assert np.array_equal(out_p, out[perm])


def test_gemm_stages_and_combine_match_numpy(orc):
    rng = np.random.default_rng(22)
    T, H, I, E, k = 10, 64, 32, 4, 2
    xb = _rand_bf16(rng, (T, H))
    w13 = _rand_bf16(rng, (E, 2 * I, H), H ** -0.5)
    w2 = _rand_bf16(rng, (E, H, I), I ** -0.5)
    tok = rng.integers(0, T, 17)
    ex = rng.integers(0, E, 17).astype(np.int32)
    act = orc.gemm1_bf16_rows(xb, w13, tok, ex)
    xv, g13, g2 = _bits_to_f64(xb), _bits_to_f64(w13), _bits_to_f64(w2)
    for n in range(17):
        g = g13[ex[n], :I] @ xv[tok[n]]
        u = g13[ex[n], I:] @ xv[tok[n]]
        assert np.allclose(act[n], _silu(g) * u, rtol=1e-12, atol=1e-14)
    ab = _rand_bf16(rng, (23, I))
    rows = rng.integers(0, 23, 9)
    ex2 = rng.integers(0, E, 9).astype(np.int32)
    y = orc.gemm2_bf16_rows(ab, w2, rows, ex2)
    av = _bits_to_f64(ab)
    for n in range(9):
        assert np.allclose(y[n], g2[ex2[n]] @ av[rows[n]], rtol=1e-12, atol=1e-14)
    # combine
    R = T * k
    yb = _rand_bf16(rng, (R, H))
    wt = rng.uniform(0, 1, (T, k)).astype(np.float32)
    a2r = rng.permutation(R).astype(np.int32)
    out, outb = orc.combine(yb, wt, a2r)
    yv = _bits_to_f64(yb)
    ref = np.einsum("tj,tjh->th", wt.astype(np.float64), yv[a2r.reshape(T, k)])
    assert np.allclose(out, ref, rtol=1e-14, atol=1e-15)
    # one bf16 rounding of the fp64 sum: within half a bf16 ulp (2^-8 relative)
    ob = _bits_to_f64(outb)
    assert np.all(np.abs(ob - out) <= np.abs(out) * 2.0 ** -8 + 1e-300)


def _fp8_case(orc, rng, T=6, H=256, I=128, E=4, k=2):
    xb = _rand_bf16(rng, (T, H))
    w13 = _rand_bf16(rng, (E, 2 * I, H), H ** -0.5)
    w2 = _rand_bf16(rng, (E, H, I), I ** -0.5)
    w13p, w13sf = orc.quant_mxfp4(w13)
    w2p, w2sf = orc.quant_mxfp4(w2)
    lg = rng.standard_normal((T, E)).astype(np.float32)
    ids, w = orc.route(lg, k)
    return xb, w13p, w13sf, w2p, w2sf, ids, w


def test_fp8_path_without_requant_reduces_to_bf16_path(orc):
    """Dequantised e4m3 activations and MXFP4 weights are exact bf16 values, so the
    block-scaled oracle (requant off) must equal the BF16 oracle on them bit for bit."""
    rng = np.random.default_rng(30)
    xb, w13p, w13sf, w2p, w2sf, ids, w = _fp8_case(orc, rng)
    out8, _ = orc.forward_fp8_mxfp4(xb, ids, w, w13p, w13sf, w2p, w2sf, requant_act=False)
    xq, sx = orc.quant_fp8_bf16(xb)
    xdeq = orc.e4m3_decode(xq) * np.repeat(sx.astype(np.float64), 128, axis=1)
    w13d = orc.mxfp4_dequant(w13p, w13sf)
    w2d = orc.mxfp4_dequant(w2p, w2sf)
    to_bits = lambda a: _bf16_bits(a.astype(np.float32))
    for a in (xdeq, w13d, w2d):           # exactness of the bf16 re-encoding
        assert np.array_equal(_bits_to_f64(to_bits(a)), a)
    out16, _ = orc.forward_bf16(to_bits(xdeq), ids, w, to_bits(w13d), to_bits(w2d))
    assert np.array_equal(out8, out16)


def test_fp8_path_with_requant_matches_numpy_composition(orc):
    rng = np.random.default_rng(31)
    xb, w13p, w13sf, w2p, w2sf, ids, w = _fp8_case(orc, rng)
    out, _ = orc.forward_fp8_mxfp4(xb, ids, w, w13p, w13sf, w2p, w2sf, requant_act=True)
    xq, sx = orc.quant_fp8_bf16(xb)
    xdeq = orc.e4m3_decode(xq) * np.repeat(sx.astype(np.float64), 128, axis=1)
    w13d = orc.mxfp4_dequant(w13p, w13sf)
    w2d = orc.mxfp4_dequant(w2p, w2sf)
    I = w13d.shape[1] // 2
    T, k = ids.shape
    ref = np.zeros((T, xb.shape[1]))
    for t in range(T):
        for j in range(k):
            e = ids[t, j]
            a = _silu(w13d[e, :I] @ xdeq[t]) * (w13d[e, I:] @ xdeq[t])
            s = np.array([2.0 ** math.ceil(math.log2(np.abs(a[g:g + 128]).max() / 448.0))
                          for g in range(0, I, 128)])
            aq = torch.tensor((a / np.repeat(s, 128)).astype(np.float32)).to(
                torch.float8_e4m3fn).to(torch.float64).numpy() * np.repeat(s, 128)
            ref[t] += w[t, j] * (w2d[e] @ aq)
    assert np.allclose(out, ref, rtol=1e-11, atol=1e-13)
    # the row-stage functions compose to the same thing
    tok = np.repeat(np.arange(T), k)
    ex = ids.reshape(-1)
    act = orc.gemm1_fp8_rows(xq, sx, w13p, w13sf, tok, ex, requant_act=True)
    aq, sa = orc.quant_fp8(act)
    assert np.array_equal(orc.e4m3_decode(aq) * np.repeat(sa, 128, 1), act)
    y = orc.gemm2_fp8_rows(aq, sa, w2p, w2sf, np.arange(T * k), ex)
    comb = (w.reshape(-1, 1) * y).reshape(T, k, -1).sum(1)
    assert np.allclose(comb, out, rtol=1e-12, atol=1e-14)
