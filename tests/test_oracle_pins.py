"""Pins of the fp64 oracle against facts that do not come from the oracle itself.

The pages ("MTP1 Post-Portfolio Eager-Cycle Profile", table "Post-Portfolio Device
Attribution"; "row/QUANT-CT-MXFP4-C8-DIFF") name the layer's steps but print no
worked values, so every pin here is a published table, a closed form worked by
hand, a library routine on a special case, brute force, or an exact invariant.
Each is chosen so that a plausible slip in the oracle (nibble order, gate/up
order, a clamp bound, a sign, a scale offset, a transposed matrix, a dropped
renormalisation, an unstable permutation) fails at least one of them.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import scipy.special

import oracle
from moe_inputs import generator as gen

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _e2m1_table():
    vals = {}
    with open(os.path.join(GOLDEN, "e2m1_ocp_mx_v1.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                c, v = line.split()
                vals[int(c)] = float(v)
    assert sorted(vals) == list(range(16))
    return np.array([vals[c] for c in range(16)])


E2M1 = _e2m1_table()

# every finite bf16 value, for brute-force nearest rounding
_ALL_BF16 = (np.arange(65536, dtype=np.uint32) << 16).view(np.float32)
_BF16_VALS = np.unique(_ALL_BF16[np.isfinite(_ALL_BF16)].astype(np.float64))


def bf16_nearest(v: float) -> float:
    """Brute force: the nearest finite bf16 value to v, ties to the even bit pattern."""
    i = np.searchsorted(_BF16_VALS, v)
    cands = [_BF16_VALS[j] for j in (i - 1, i) if 0 <= j < len(_BF16_VALS)]
    fv = Fraction(v)
    best = min(abs(Fraction(c) - fv) for c in cands)
    ties = [c for c in cands if abs(Fraction(c) - fv) == best]
    if len(ties) == 1:
        return ties[0]
    even = [c for c in ties if (int(np.float32(c).view(np.uint32)) >> 16) % 2 == 0]
    return even[0]


def decode_np(q: np.ndarray, s: np.ndarray) -> np.ndarray:
    """Dequantise an MXFP4 matrix with the OCP table fixture (independent of the oracle)."""
    lo = E2M1[q & 15]
    hi = E2M1[q >> 4]
    vals = np.empty(q.shape[:-1] + (q.shape[-1] * 2,))
    vals[..., 0::2] = lo
    vals[..., 1::2] = hi
    scale = np.repeat(2.0 ** (s.astype(np.float64) - 127.0), 32, axis=-1)
    return vals * scale


def bf16_of_bits(bits):
    return gen.bf16_bits_to_f64(np.asarray(bits, dtype=np.uint16))


def bits_of_bf16(v: float) -> int:
    return int(np.float32(v).view(np.uint32)) >> 16


# ----------------------------------------------------------------------------- formats

def test_e2m1_matches_ocp_table():
    for c in range(16):
        v = oracle.e2m1_value(c)
        assert v == E2M1[c]
        assert math.copysign(1.0, v) == math.copysign(1.0, E2M1[c])   # code 8 is -0


def test_e8m0_scale_is_power_of_two():
    for b in range(255):
        assert oracle.e8m0_scale(b) == 2.0 ** (b - 127)
    assert math.isnan(oracle.e8m0_scale(255))


def test_nibble_order_and_scale_blocks():
    # one row, K = 64: byte 0 = 0x21 -> k0 = code 1 (0.5), k1 = code 2 (1.0);
    # byte 16 = 0x9F -> k32 = code 15 (-6), k33 = code 9 (-0.5); scales 127 then 128.
    q = np.zeros((1, 32), np.uint8)
    q[0, 0] = 0x21
    q[0, 16] = 0x9F
    s = np.array([[127, 128]], np.uint8)
    assert oracle.mxfp4_weight(q, s, 0, 0) == 0.5
    assert oracle.mxfp4_weight(q, s, 0, 1) == 1.0
    assert oracle.mxfp4_weight(q, s, 0, 2) == 0.0
    assert oracle.mxfp4_weight(q, s, 0, 32) == -12.0
    assert oracle.mxfp4_weight(q, s, 0, 33) == -1.0


def test_dequant_brute_force_all_bytes():
    for sb in (0, 1, 120, 121, 122, 123, 124, 200, 254):
        q = np.arange(256, dtype=np.uint8).reshape(16, 16)
        s = np.full((16, 1), sb, np.uint8)
        ref = decode_np(q, s)
        for r in range(16):
            for kk in range(32):
                assert oracle.mxfp4_weight(q, s, r, kk) == ref[r, kk]


def test_scaled_e2m1_exact_in_bf16():
    # every E2M1 value times 2^(e-127), e in the workloads' range {120..124}, is a bf16 value
    for e in range(120, 125):
        for c in range(16):
            v = E2M1[c] * 2.0 ** (e - 127)
            assert bf16_of_bits(oracle.round_bf16(v)) == v


def test_round_bf16_brute_force():
    rng = np.random.default_rng(7)
    vals = list(rng.standard_normal(3000) * 10.0 ** rng.integers(-6, 6, 3000))
    # exact midpoints between adjacent bf16 values: ties must go to the even pattern
    for b in (0x3F80, 0x3F81, 0x4049, 0x404A, 0xC2F7, 0x0081):
        lo = float(bf16_of_bits(b))
        hi = float(bf16_of_bits(b + 1))
        vals.append((lo + hi) / 2)
    vals += [0.0, -0.0, 2.0 ** -130, -(2.0 ** -131) * 3, 3.3895313892515355e38]
    for v in vals:
        got = bf16_of_bits(oracle.round_bf16(v))
        want = bf16_nearest(v)
        assert got == want, (v, got, want)


# ----------------------------------------------------------------------------- hand-worked example

def _hand_example():
    """M=1, H=I=32, E=k=2; every value below is worked by hand (see the test's comments)."""
    H = I = 32
    x = np.full((1, H), bits_of_bf16(0.25), np.uint16)
    wr = np.zeros((2, H), np.float32)
    wr[0] = 0.125                                     # logits (1, 0)
    w13q = np.zeros((2, 2 * I, H // 2), np.uint8)
    w13s = np.zeros((2, 2 * I, H // 32), np.uint8)
    w2q = np.zeros((2, H, I // 2), np.uint8)
    w2s = np.zeros((2, H, I // 32), np.uint8)
    # expert 0: gate and up all code 2 (1.0) at scale 127; w2 all code 1 (0.5) at scale 127
    w13q[0] = 0x22
    w13s[0] = 127
    w2q[0] = 0x11
    w2s[0] = 127
    # expert 1: gate code 1 (0.5) at scale 126 -> 0.25; up code 10 (-1.0) at 127; w2 code 3 (1.5) at 128 -> 3.0
    w13q[1, :I] = 0x11
    w13s[1, :I] = 126
    w13q[1, I:] = 0xAA
    w13s[1, I:] = 127
    w2q[1] = 0x33
    w2s[1] = 128
    return x, wr, w13q, w13s, w2q, w2s


def test_hand_worked_example():
    x, wr, w13q, w13s, w2q, w2s = _hand_example()
    r = oracle.forward(x, wr, None, w13q, w13s, w2q, w2s, k=2)
    e = math.e
    assert r["topk_ids"].tolist() == [[0, 1]]
    assert r["topk_w"][0, 0] == pytest.approx(e / (e + 1), rel=1e-15)
    assert r["topk_w"][0, 1] == pytest.approx(1 / (e + 1), rel=1e-15)
    # expert 0: g = u = 32*0.25*1.0 = 8 -> both clamp to 7 -> h = bf16(7*sigmoid(7)*7) = bf16(48.955...) = 49
    # expert 1: g = 32*0.25*0.25 = 2, u = -8 -> -7 -> h = bf16(-7 * 2*sigmoid(2)) = bf16(-12.331...) = -12.3125
    h = bf16_of_bits(r["h"])
    assert np.all(h[0] == 49.0)
    assert np.all(h[1] == -12.3125)
    # y0 = 32 * 0.5 * 49 = 784; y1 = 32 * 3.0 * -12.3125 = -1182
    want = 784.0 * e / (e + 1) - 1182.0 / (e + 1)
    assert want == pytest.approx(255.26116558658964, rel=1e-15)
    assert np.allclose(r["out64"], want, rtol=1e-14, atol=0)
    assert np.all(bf16_of_bits(r["out_bf16"]) == 255.0)


# ----------------------------------------------------------------------------- router

def _np_logits(x_bits, wr, bias):
    lg = bf16_of_bits(x_bits) @ wr.astype(np.float64).T
    return lg if bias is None else lg + bias.astype(np.float64)


@pytest.mark.parametrize("ci", [0, 1, 4])
def test_router_against_sort_and_softmax(ci):
    shape = gen.CONFIGS[ci]
    M = min(shape.default_M, 64)
    inp = gen.make_inputs(ci, M, weights="none")
    ids, w, logits = oracle.route(inp.x, inp.router_w, inp.router_bias, shape.k)
    ref = _np_logits(inp.x, inp.router_w, inp.router_bias)
    assert np.allclose(logits, ref, rtol=1e-12, atol=1e-12)
    order = np.argsort(-ref, axis=1, kind="stable")[:, :shape.k]
    assert np.array_equal(ids, order)
    assert np.all(np.abs(w.sum(axis=1) - 1.0) <= 1e-12)
    p = scipy.special.softmax(ref, axis=1)
    sel = np.take_along_axis(p, order, axis=1)
    assert np.allclose(w, sel / sel.sum(axis=1, keepdims=True), rtol=1e-12)
    assert np.all(np.diff(w, axis=1) <= 0)             # slots in descending weight


def test_router_k_equals_e_is_plain_softmax():
    inp = gen.make_inputs(0, 2, weights="none")
    E = inp.router_w.shape[0]
    ids, w, _ = oracle.route(inp.x, inp.router_w, None, E)
    lg = _np_logits(inp.x, inp.router_w, None)
    p = scipy.special.softmax(lg, axis=1)
    assert np.allclose(np.take_along_axis(p, ids, axis=1), w, rtol=1e-12)


def test_router_ties_go_to_lower_id():
    x = np.zeros((3, 64), np.uint16)                    # all logits 0
    wr = np.ones((8, 64), np.float32)
    ids, w, _ = oracle.route(x, wr, None, 3)
    assert ids.tolist() == [[0, 1, 2]] * 3
    assert np.allclose(w, 1 / 3, rtol=1e-15)


def test_router_bias_enters_logits():
    inp = gen.make_inputs(0, 2, weights="none")
    E = inp.router_w.shape[0]
    bias = np.zeros(E, np.float32)
    bias[E - 1] = 100.0
    ids, w, lg = oracle.route(inp.x, inp.router_w, bias, 4)
    assert np.all(ids[:, 0] == E - 1)
    assert np.allclose(lg, _np_logits(inp.x, inp.router_w, bias), rtol=1e-12)
    assert np.all(w[:, 0] > 0.999)


def test_generator_margin_holds():
    for ci, M in ((1, 8), (2, 32), (4, 1024)):
        inp = gen.make_inputs(ci, M, weights="none")
        lg = _np_logits(inp.x, inp.router_w, inp.router_bias)
        top = -np.sort(-lg, axis=1)[:, :inp.shape.k + 1]
        assert np.all(top[:, :-1] - top[:, 1:] >= 1e-4)


# ----------------------------------------------------------------------------- permutation

@pytest.mark.parametrize("ci", [0, 1, 4])
def test_permute_invariants(ci):
    shape = gen.CONFIGS[ci]
    inp = gen.make_inputs(ci, shape.default_M, weights="none")
    ids, _, _ = oracle.route(inp.x, inp.router_w, inp.router_bias, shape.k)
    off, srt, inv = oracle.permute(ids, shape.E)
    flat = ids.ravel()
    n = flat.size
    assert off[0] == 0 and off[-1] == n and np.all(np.diff(off) >= 0)
    assert np.array_equal(np.diff(off), np.bincount(flat, minlength=shape.E))
    assert np.array_equal(np.sort(srt), np.arange(n))
    assert np.array_equal(srt, np.argsort(flat, kind="stable"))
    for e in range(shape.E):
        seg = srt[off[e]:off[e + 1]]
        assert np.all(flat[seg] == e)
        assert np.all(np.diff(seg) > 0)
    assert np.array_equal(srt[inv], np.arange(n))


def test_skewed_routing_is_skewed():
    inp = gen.make_inputs(4, 1024, weights="none")
    ids, _, _ = oracle.route(inp.x, inp.router_w, inp.router_bias, 8)
    counts = np.bincount(ids.ravel(), minlength=128)
    assert counts[:4].min() > 500                      # a few experts take hundreds of rows
    assert (counts <= 2).sum() > 64                    # many take 0-2


# ----------------------------------------------------------------------------- layer special cases

def _bf16_nearest_vec(v):
    return np.array([bf16_nearest(float(a)) for a in v])


def test_single_expert_reduces_to_dense_mlp():
    # E = k = 1, H != I so that a transposed operand cannot pass
    H, I = 96, 64
    rng = np.random.default_rng(3)
    x = gen._bf16_bits_rne(rng.standard_normal((2, H)))
    wr = np.ones((1, H), np.float32)
    w13q = rng.integers(0, 256, (1, 2 * I, H // 2), dtype=np.uint8)
    w13s = rng.integers(123, 127, (1, 2 * I, H // 32), dtype=np.uint8)
    w2q = rng.integers(0, 256, (1, H, I // 2), dtype=np.uint8)
    w2s = rng.integers(120, 125, (1, H, I // 32), dtype=np.uint8)
    r = oracle.forward(x, wr, None, w13q, w13s, w2q, w2s, k=1)
    W13 = decode_np(w13q[0], w13s[0])
    W2 = decode_np(w2q[0], w2s[0])
    assert W13.shape == (2 * I, H) and W2.shape == (H, I)
    for t in range(2):
        xv = bf16_of_bits(x[t])
        g = W13[:I] @ xv
        u = W13[I:] @ xv
        # the clamps are exercised: g above 7 (clamped) and below -7 (not clamped: silu's
        # negative tail is kept), u beyond both bounds
        assert g.max() > 7 and g.min() < -7 and u.max() > 7 and u.min() < -7
        a = np.minimum(g, 7.0)
        hv = _bf16_nearest_vec(a * scipy.special.expit(a) * np.clip(u, -7.0, 7.0))
        assert np.array_equal(bf16_of_bits(r["h"][t]), hv)
        y = W2 @ hv
        assert np.allclose(r["out64"][t], y, rtol=1e-12, atol=1e-12)
        assert np.array_equal(bf16_of_bits(r["out_bf16"][t]), _bf16_nearest_vec(y))
    assert r["topk_w"][0, 0] == 1.0


def _small_layer(ci=0):
    inp = gen.make_inputs(ci, gen.CONFIGS[ci].default_M)
    return inp


def test_down_scale_plus_one_doubles_output_exactly():
    inp = _small_layer()
    k = inp.shape.k
    a = oracle.forward(inp.x, inp.router_w, None, inp.w13_q, inp.w13_s, inp.w2_q, inp.w2_s, k)
    b = oracle.forward(inp.x, inp.router_w, None, inp.w13_q, inp.w13_s, inp.w2_q, inp.w2_s + 1, k)
    assert np.array_equal(b["out64"], 2.0 * a["out64"])
    assert np.array_equal(bf16_of_bits(b["out_bf16"]), 2.0 * bf16_of_bits(a["out_bf16"]))
    assert np.array_equal(a["h"], b["h"])


def test_relabelled_experts_give_identical_output():
    inp = _small_layer()
    E, k = inp.shape.E, inp.shape.k
    perm = np.random.default_rng(1).permutation(E)
    a = oracle.forward(inp.x, inp.router_w, None, inp.w13_q, inp.w13_s, inp.w2_q, inp.w2_s, k)
    b = oracle.forward(inp.x, inp.router_w[perm], None, inp.w13_q[perm], inp.w13_s[perm],
                       inp.w2_q[perm], inp.w2_s[perm], k)
    assert np.array_equal(perm[b["topk_ids"]], a["topk_ids"])
    # the softmax denominator is summed in expert-id order, so weights move by fp64 ulps only
    assert np.allclose(a["out64"], b["out64"], rtol=1e-13, atol=1e-13)
    assert np.array_equal(a["h"], b["h"])


def test_token_permutation_permutes_rows():
    inp = gen.make_inputs(1, 4)
    k = inp.shape.k
    perm = np.array([2, 0, 3, 1])
    a = oracle.forward(inp.x, inp.router_w, None, inp.w13_q, inp.w13_s, inp.w2_q, inp.w2_s, k)
    b = oracle.forward(inp.x[perm], inp.router_w, None, inp.w13_q, inp.w13_s, inp.w2_q, inp.w2_s, k)
    assert np.array_equal(b["out64"], a["out64"][perm])
    assert np.array_equal(b["topk_ids"], a["topk_ids"][perm])


def test_token_subset_matches_full_forward():
    inp = gen.make_inputs(1, 8)
    k = inp.shape.k
    a = oracle.forward(inp.x, inp.router_w, None, inp.w13_q, inp.w13_s, inp.w2_q, inp.w2_s, k)
    toks = [5, 1]
    need = set(a["topk_ids"][toks].ravel().tolist())
    experts = {e: inp.expert_weights(e) for e in need}
    b = oracle.forward(inp.x, inp.router_w, None,
                       {e: v[0] for e, v in experts.items()}, {e: v[1] for e, v in experts.items()},
                       {e: v[2] for e, v in experts.items()}, {e: v[3] for e, v in experts.items()},
                       k, tokens=toks, I=inp.shape.I)
    assert np.array_equal(b["out64"][toks], a["out64"][toks])


def test_per_expert_regeneration_matches_full_arrays():
    inp = gen.make_inputs(0, 2)
    for e in (0, 5, 15):
        q13, s13, q2, s2 = inp.expert_weights(e)
        assert np.array_equal(q13, inp.w13_q[e]) and np.array_equal(s13, inp.w13_s[e])
        assert np.array_equal(q2, inp.w2_q[e]) and np.array_equal(s2, inp.w2_s[e])


def test_swiglu_step_matches_forward_h():
    inp = _small_layer()
    k = inp.shape.k
    a = oracle.forward(inp.x, inp.router_w, None, inp.w13_q, inp.w13_s, inp.w2_q, inp.w2_s, k)
    t, j = 1, 2
    e = a["topk_ids"][t, j]
    g, u, h = oracle.expert_swiglu(inp.x[t], inp.w13_q[e], inp.w13_s[e])
    assert np.array_equal(h, a["h"][t * k + j])
    W13 = decode_np(inp.w13_q[e], inp.w13_s[e])
    xv = bf16_of_bits(inp.x[t])
    assert np.allclose(g, W13[:inp.shape.I] @ xv, rtol=1e-12, atol=1e-12)
    assert np.allclose(u, W13[inp.shape.I:] @ xv, rtol=1e-12, atol=1e-12)
