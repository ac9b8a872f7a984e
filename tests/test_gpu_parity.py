"""GPU parity of every step of the layer against the fp64 oracle, through the C ABI.

Small workloads are compared element by element on every output; the full-size
DeepSeek-class workloads (6 GB of MXFP4 weights) are compared on the complete
routing and permutation and on sampled tokens' outputs, with the weights
generated on the device from the same counter streams the oracle regenerates on
the host.
"""
import numpy as np
import pytest
import torch

import oracle
from moe_inputs import generator as gen
from tests import _gpu_util as U

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


@pytest.fixture(scope="module")
def moe():
    import decode_moe_layer_b200 as m
    return m


def _gpu_route(moe, d, k):
    ids, w = moe.moe_route(d["x"], d["router_w"], k, router_bias=d["router_bias"])
    torch.cuda.synchronize()
    return ids.cpu().numpy(), w.cpu().numpy()


# ----------------------------------------------------------------------------- router + permutation

ROUTE_CASES = [(0, 2), (1, 1), (1, 8), (2, 1), (2, 32), (3, 512), (4, 1024), (1, 37)]


@pytest.mark.parametrize("ci,M", ROUTE_CASES)
def test_route_and_permute_bit_exact(moe, ci, M):
    inp = gen.make_inputs(ci, M, weights="none")
    k, E = inp.shape.k, inp.shape.E
    d = {"x": U.bits_to_bf16_tensor(inp.x), "router_w": torch.from_numpy(inp.router_w).cuda(),
         "router_bias": None if inp.router_bias is None else torch.from_numpy(inp.router_bias).cuda()}
    ids, w = _gpu_route(moe, d, k)
    rids, rw, _ = oracle.route(inp.x, inp.router_w, inp.router_bias, k)
    assert np.array_equal(ids, rids)
    assert np.abs(w - rw).max() <= U.W_TOL
    off, srt, inv = moe.moe_permute(torch.from_numpy(ids).cuda(), E)
    roff, rsrt, rinv = oracle.permute(rids, E)
    assert np.array_equal(off.cpu().numpy(), roff)
    assert np.array_equal(srt.cpu().numpy(), rsrt)
    assert np.array_equal(inv.cpu().numpy(), rinv)


def test_route_ties_and_all_experts(moe):
    # all-zero x: every logit ties -> experts 0..k-1 with weight 1/k
    x = torch.zeros((5, 256), dtype=torch.bfloat16, device="cuda")
    wr = torch.randn((16, 256), device="cuda")
    ids, w = moe.moe_route(x, wr, 4)
    assert ids.cpu().tolist() == [[0, 1, 2, 3]] * 5
    assert torch.allclose(w.cpu(), torch.full((5, 4), 0.25), atol=0, rtol=0)
    # k == E: every expert selected, weights are the plain softmax
    inp = gen.make_inputs(0, 2, weights="none")
    E = inp.shape.E
    ids, w = moe.moe_route(U.bits_to_bf16_tensor(inp.x), torch.from_numpy(inp.router_w).cuda(), E)
    rids, rw, _ = oracle.route(inp.x, inp.router_w, None, E)
    assert np.array_equal(ids.cpu().numpy(), rids)
    assert np.abs(w.cpu().numpy() - rw).max() <= U.W_TOL


def test_permute_edge_cases(moe):
    E = 64
    rng = np.random.default_rng(0)
    for M, k in [(1, 1), (1, 8), (3, 5), (2048, 8), (511, 32)]:
        ids = np.stack([rng.choice(E, k, replace=False) for _ in range(M)]).astype(np.int32)
        if M == 2048:
            ids[:] = np.arange(k)        # every assignment on the first k experts
        off, srt, inv = moe.moe_permute(torch.from_numpy(ids).cuda(), E)
        roff, rsrt, rinv = oracle.permute(ids, E)
        assert np.array_equal(off.cpu().numpy(), roff), (M, k)
        assert np.array_equal(srt.cpu().numpy(), rsrt), (M, k)
        assert np.array_equal(inv.cpu().numpy(), rinv), (M, k)
    # tokens that repeat an expert (the token-mask ranking must hand over to the exact one), and
    # masks too large for shared memory (E * ceil(M/32) words above 64 KB)
    for M, k, E2, repeat in [(300, 4, 16, True), (700, 2, 1024, False)]:
        if repeat:
            ids = rng.integers(0, E2, size=(M, k)).astype(np.int32)
            assert any(len(set(r)) < k for r in ids.tolist())
        else:
            ids = np.stack([rng.choice(E2, k, replace=False) for _ in range(M)]).astype(np.int32)
        off, srt, inv = moe.moe_permute(torch.from_numpy(ids).cuda(), E2)
        roff, rsrt, rinv = oracle.permute(ids, E2)
        assert np.array_equal(off.cpu().numpy(), roff), (M, k, E2)
        assert np.array_equal(srt.cpu().numpy(), rsrt), (M, k, E2)
        assert np.array_equal(inv.cpu().numpy(), rinv), (M, k, E2)


# ----------------------------------------------------------------------------- gate_up + clamp-SwiGLU

@pytest.mark.parametrize("ci,M", [(0, 2), (1, 8), (1, 37), (1, 96), (2, 1), (2, 16)])
def test_gate_up_swiglu(moe, ci, M):
    big = ci >= 2
    inp = gen.make_inputs(ci, M, weights="torch" if big else "numpy", device="cuda")
    k, E = inp.shape.k, inp.shape.E
    d = U.device_inputs(inp)
    rids, rw, _ = oracle.route(inp.x, inp.router_w, inp.router_bias, k)
    roff, rsrt, rinv = oracle.permute(rids, E)
    h = moe.moe_gate_up_swiglu(d["x"], d["w13_q"], d["w13_s"], torch.from_numpy(roff).cuda(),
                               torch.from_numpy(rsrt).cuda(), k)
    torch.cuda.synchronize()
    h_flat = U.bf16_tensor_to_f64(h)[rinv]   # flat order t*k+j
    toks = list(range(M)) if not big else [0, M - 1]
    for t in toks:
        for j in range(k):
            e = int(rids[t, j])
            q13, s13 = (inp.w13_q[e], inp.w13_s[e]) if not big else inp.expert_weights(e)[:2]
            g, u, hb = oracle.expert_swiglu(inp.x[t], q13, s13)
            U.check_h_bound(h_flat[t * k + j], hb, g, u, inp.x[t], q13, s13, "c%d M=%d h[t=%d,j=%d]" % (ci, M, t, j))
    flips = sum(f for w, f, n in U.FLIP_LOG if w.startswith("c%d M=%d " % (ci, M)))
    total = sum(n for w, f, n in U.FLIP_LOG if w.startswith("c%d M=%d " % (ci, M)))
    print("h rounding flips vs the fp64 oracle: %d of %d (%.2f%%)" % (flips, total, 100.0 * flips / total))


# ----------------------------------------------------------------------------- down + combine

@pytest.mark.parametrize("ci,M", [(0, 2), (1, 8), (1, 37), (1, 96)])
def test_down_combine(moe, ci, M):
    inp = gen.make_inputs(ci, M)
    k, E = inp.shape.k, inp.shape.E
    d = U.device_inputs(inp)
    r = U.oracle_forward(inp)
    rids, rw = r["topk_ids"], r["topk_w"]
    roff, rsrt, rinv = oracle.permute(rids, E)
    h_bits = r["h"][rsrt]                                         # oracle h in expert-grouped order
    hb = U.bits_to_bf16_tensor(h_bits)
    out = moe.moe_down_combine(hb, d["w2_q"], d["w2_s"], torch.from_numpy(rw.astype(np.float32)).cuda(),
                               torch.from_numpy(roff).cuda(), torch.from_numpy(rsrt).cuda(), M, k)
    torch.cuda.synchronize()
    U.check_out(U.bf16_tensor_to_f64(out), r["out64"], "down_combine c%d M=%d" % (ci, M))


# ----------------------------------------------------------------------------- whole layer

# (1, 96): M*k >= 6E, so 16-assignment tiles (two MMA n-tiles per decoded weight fragment)
SMALL_FORWARD = [(0, 2), (1, 1), (1, 2), (1, 4), (1, 8), (1, 37), (1, 96)]


@pytest.mark.parametrize("ci,M", SMALL_FORWARD)
def test_forward_small_full_compare(moe, ci, M):
    inp = gen.make_inputs(ci, M)
    d = U.device_inputs(inp)
    k = inp.shape.k
    ws = torch.empty(moe.moe_workspace_bytes(M, inp.shape.H, inp.shape.I, inp.shape.E, k), dtype=torch.uint8,
                     device="cuda")
    ids = torch.empty((M, k), dtype=torch.int32, device="cuda")
    tw = torch.empty((M, k), dtype=torch.float32, device="cuda")
    st = torch.full((1,), 123, dtype=torch.int32, device="cuda")
    out = moe.moe_mxfp4_forward_ex(d["x"], d["router_w"], d["w13_q"], d["w13_s"], d["w2_q"], d["w2_s"], k, ws,
                                   router_bias=d["router_bias"], topk_ids_out=ids, topk_w_out=tw, status_out=st)
    torch.cuda.synchronize()
    assert int(st.item()) == moe.MOE_OK
    r = U.oracle_forward(inp)
    assert np.array_equal(ids.cpu().numpy(), r["topk_ids"])
    assert np.abs(tw.cpu().numpy() - r["topk_w"]).max() <= U.W_TOL
    U.check_out(U.bf16_tensor_to_f64(out), r["out64"], "forward c%d M=%d" % (ci, M))
    # the 13-argument form (library workspace, no bias) gives the same bytes here
    out2 = moe.moe_mxfp4_forward(d["x"], d["router_w"], d["w13_q"], d["w13_s"], d["w2_q"], d["w2_s"], k)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), out2.view(torch.int16))


LARGE_FORWARD = [(2, 1), (2, 2), (2, 8), (2, 16), (2, 32), (3, 256), (3, 512), (4, 1024)]


@pytest.fixture(scope="module")
def large_weights():
    cache = {}

    def get(ci, M):
        key = ci
        shape = gen.CONFIGS[ci]
        seed = gen.config_seed(ci, M)
        if key not in cache or cache[key][0] != seed:
            cache.clear()
            torch.cuda.empty_cache()
            inp = gen.make_inputs(ci, M, weights="torch", device="cuda")
            cache[key] = (seed, inp)
        return cache[key][1]
    yield get
    cache.clear()
    torch.cuda.empty_cache()


@pytest.mark.parametrize("ci,M", LARGE_FORWARD)
def test_forward_large_sampled(moe, large_weights, ci, M):
    inp = large_weights(ci, M)
    d = U.device_inputs(inp)
    k = inp.shape.k
    ids = torch.empty((M, k), dtype=torch.int32, device="cuda")
    tw = torch.empty((M, k), dtype=torch.float32, device="cuda")
    ws = torch.empty(moe.moe_workspace_bytes(M, inp.shape.H, inp.shape.I, inp.shape.E, k), dtype=torch.uint8,
                     device="cuda")
    out = moe.moe_mxfp4_forward_ex(d["x"], d["router_w"], d["w13_q"], d["w13_s"], d["w2_q"], d["w2_s"], k, ws,
                                   router_bias=d["router_bias"], topk_ids_out=ids, topk_w_out=tw)
    torch.cuda.synchronize()
    rids, rw, _ = oracle.route(inp.x, inp.router_w, inp.router_bias, k)
    assert np.array_equal(ids.cpu().numpy(), rids)                 # whole routing, bit-exact
    assert np.abs(tw.cpu().numpy() - rw).max() <= U.W_TOL
    # every token when M <= 64; else at least 64 that cover every mma.sync tile slot and fill
    # count, the first and last assignment of tensor-core tiles, and random ones
    toks, desc = U.sample_tokens(rids, inp.shape.E, inp.shape.H, inp.shape.I, seed=M)
    print("c%d M=%d compared: %s" % (ci, M, desc))
    r = U.oracle_forward(inp, tokens=toks)
    got = U.bf16_tensor_to_f64(out)
    U.check_out(got[toks], r["out64"][toks], "forward c%d M=%d (%s)" % (ci, M, desc))
    assert np.all(np.isfinite(got))


# ----------------------------------------------------------------------------- tensor-core tiles, step by step

WIDE_STEP_SHAPES = [
    (1024, 512, 4, 2, 80),    # ~40 assignments per expert: tensor-core tiles for every expert
    (512, 1024, 16, 4, 160),  # ~40 per expert, spread: tensor-core and mma.sync tiles in one call
]


@pytest.mark.parametrize("H,I,E,k,M", WIDE_STEP_SHAPES)
def test_gate_up_and_down_steps_on_tensor_core_tiles(moe, H, I, E, k, M):
    # the step entry points take the same tile split as the whole layer, wide tiles included
    assert U.wide_path_on(M, H, I, E, k)
    shape = gen.LayerShape("wide_step", H, I, E, k, (M,))
    inp = gen.make_inputs(0, M, shape=shape, seed=3 * H + I + E + k + M)
    d = U.device_inputs(inp)
    r = U.oracle_forward(inp)
    rids, rw = r["topk_ids"], r["topk_w"]
    roff, rsrt, rinv = oracle.permute(rids, E)
    assert np.diff(roff).max() >= U.WIDE_MIN_TOKENS
    h = moe.moe_gate_up_swiglu(d["x"], d["w13_q"], d["w13_s"], torch.from_numpy(roff).cuda(),
                               torch.from_numpy(rsrt).cuda(), k)
    torch.cuda.synchronize()
    h_flat = U.bf16_tensor_to_f64(h)[rinv]
    for t in range(M):
        for j in range(k):
            e = int(rids[t, j])
            g, u, hb = oracle.expert_swiglu(inp.x[t], inp.w13_q[e], inp.w13_s[e])
            U.check_h_bound(h_flat[t * k + j], hb, g, u, inp.x[t], inp.w13_q[e], inp.w13_s[e],
                            "wide step %s h[t=%d,j=%d]" % ((H, I, E, k, M), t, j))
    out = moe.moe_down_combine(U.bits_to_bf16_tensor(r["h"][rsrt]), d["w2_q"], d["w2_s"],
                               torch.from_numpy(rw.astype(np.float32)).cuda(), torch.from_numpy(roff).cuda(),
                               torch.from_numpy(rsrt).cuda(), M, k)
    torch.cuda.synchronize()
    U.check_out(U.bf16_tensor_to_f64(out), r["out64"], "wide step down %s" % ((H, I, E, k, M),))


# ----------------------------------------------------------------------------- inputs across the bf16 range

def _wide_range_inputs(H, I, E, k, M, seed):
    """Every x row mixes magnitudes above 65504 and below 2^-17 (each element of a seeded
    workload scaled by 2^d, d uniform over -40..24: exact in bf16), and every E8M0 byte is drawn
    from 90..150 (weights from 2^-38 to 6 * 2^23)."""
    shape = gen.LayerShape("wide_range", H, I, E, k, (M,))
    inp = gen.make_inputs(0, M, shape=shape, seed=seed)
    rng = np.random.default_rng(seed)
    inp.w13_s = rng.integers(90, 151, size=inp.w13_s.shape).astype(np.uint8)
    inp.w2_s = rng.integers(90, 151, size=inp.w2_s.shape).astype(np.uint8)
    base = gen.bf16_bits_to_f64(inp.x)
    for _ in range(100):
        xv = base * np.exp2(rng.integers(-40, 25, size=base.shape).astype(np.float64))
        bits = gen._bf16_bits_rne(xv)
        if gen.margin_ok(bits, inp.router_w, inp.router_bias, k).all():
            break
    else:
        raise RuntimeError("no draw met the routing margin")
    assert np.array_equal(gen.bf16_bits_to_f64(bits), xv)
    assert (np.abs(xv) > 65504).any(axis=1).all()
    assert ((np.abs(xv) < 2.0 ** -17) & (xv != 0)).any(axis=1).all()
    inp.x = bits
    return inp


@pytest.mark.parametrize("H,I,E,k,M", [
    (1024, 512, 16, 4, 6),    # mma.sync tiles only
    (1024, 512, 4, 2, 80),    # tensor-core tiles (scale bytes above 128 take the two-multiply decode)
])
def test_wide_range_x_and_scale_bytes(moe, H, I, E, k, M):
    inp = _wide_range_inputs(H, I, E, k, M, seed=11 * H + I + E + k + M)
    d = U.device_inputs(inp)
    ids = torch.empty((M, k), dtype=torch.int32, device="cuda")
    tw = torch.empty((M, k), dtype=torch.float32, device="cuda")
    st = torch.full((1,), 123, dtype=torch.int32, device="cuda")
    ws = torch.empty(moe.moe_workspace_bytes(M, H, I, E, k), dtype=torch.uint8, device="cuda")
    out = moe.moe_mxfp4_forward_ex(d["x"], d["router_w"], d["w13_q"], d["w13_s"], d["w2_q"], d["w2_s"], k, ws,
                                   topk_ids_out=ids, topk_w_out=tw, status_out=st)
    torch.cuda.synchronize()
    assert int(st.item()) == moe.MOE_OK
    r = U.oracle_forward(inp)
    assert np.array_equal(ids.cpu().numpy(), r["topk_ids"])
    assert np.abs(tw.cpu().numpy() - r["topk_w"]).max() <= U.W_TOL
    # outputs here span many binades (x scaled by up to 2^24): the bar adds each element's own rounding
    U.check_out_heavy_tailed(U.bf16_tensor_to_f64(out), r["out64"], "wide-range forward %s" % ((H, I, E, k, M),))
    # h element by element through the step entry point
    rids = r["topk_ids"]
    roff, rsrt, rinv = oracle.permute(rids, E)
    h = moe.moe_gate_up_swiglu(d["x"], d["w13_q"], d["w13_s"], torch.from_numpy(roff).cuda(),
                               torch.from_numpy(rsrt).cuda(), k)
    torch.cuda.synchronize()
    h_flat = U.bf16_tensor_to_f64(h)[rinv]
    for t in range(M):
        for j in range(k):
            e = int(rids[t, j])
            g, u, hb = oracle.expert_swiglu(inp.x[t], inp.w13_q[e], inp.w13_s[e])
            U.check_h_bound(h_flat[t * k + j], hb, g, u, inp.x[t], inp.w13_q[e], inp.w13_s[e],
                            "wide-range h[t=%d,j=%d]" % (t, j))
