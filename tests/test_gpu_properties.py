"""Bit-exact GPU properties that need no oracle: determinism across calls and
across CUDA-graph replay (the "byte-coherent" graph check of
"row/QUANT-CT-MXFP4-C8-DIFF" and the bitwise changed-input/graph exactness gate
of "MTP1 Post-Portfolio Eager-Cycle Profile", "Decision"), exact scale
doubling, expert relabelling and token permutation, plus ragged shapes."""
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


def _fwd(moe, d, k, **kw):
    return moe.moe_mxfp4_forward(d["x"], d["router_w"], d["w13_q"], d["w13_s"], d["w2_q"], d["w2_s"], k, **kw)


def _bits(t):
    return t.view(torch.int16).cpu().numpy()


def test_repeat_calls_identical(moe):
    inp = gen.make_inputs(1, 8)
    d = U.device_inputs(inp)
    a = _fwd(moe, d, 8)
    b = _fwd(moe, d, 8)
    torch.cuda.synchronize()
    assert np.array_equal(_bits(a), _bits(b))


def test_graph_replay_matches_eager_and_follows_input(moe):
    inp = gen.make_inputs(1, 8)
    d = U.device_inputs(inp)
    k = 8
    eager = _fwd(moe, d, k)
    torch.cuda.synchronize()
    out = torch.empty_like(eager)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        _fwd(moe, d, k, out=out)          # warm the stream's workspace outside capture
        s.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            _fwd(moe, d, k, out=out)
    g.replay()
    torch.cuda.synchronize()
    assert np.array_equal(_bits(out), _bits(eager))
    # change x and the router in place (a margin-checked pair), replay: the output
    # must follow and match the oracle
    inp2 = gen.make_inputs(1, 8, seed=777)
    d["x"].copy_(U.bits_to_bf16_tensor(inp2.x))
    d["router_w"].copy_(torch.from_numpy(inp2.router_w))
    g.replay()
    torch.cuda.synchronize()
    assert not np.array_equal(_bits(out), _bits(eager))
    inp2.w13_q, inp2.w13_s, inp2.w2_q, inp2.w2_s = inp.w13_q, inp.w13_s, inp.w2_q, inp.w2_s
    r = U.oracle_forward(inp2)
    U.check_out(U.bf16_tensor_to_f64(out), r["out64"], "graph replay after x change")


def test_down_scale_plus_one_doubles_output_exactly(moe):
    inp = gen.make_inputs(0, 2)
    d = U.device_inputs(inp)
    a = _fwd(moe, d, 4)
    d2 = dict(d)
    d2["w2_s"] = d["w2_s"] + 1
    b = _fwd(moe, d2, 4)
    torch.cuda.synchronize()
    assert torch.equal(b.float(), 2.0 * a.float())


def test_expert_relabelling_identical_bytes(moe):
    inp = gen.make_inputs(1, 8)
    d = U.device_inputs(inp)
    perm = torch.from_numpy(np.random.default_rng(5).permutation(inp.shape.E)).cuda()
    d2 = {key: (v[perm].contiguous() if key in ("router_w", "w13_q", "w13_s", "w2_q", "w2_s") else v)
          for key, v in d.items()}
    a = _fwd(moe, d, 8)
    b = _fwd(moe, d2, 8)
    torch.cuda.synchronize()
    assert np.array_equal(_bits(a), _bits(b))


def test_token_permutation_permutes_rows(moe):
    inp = gen.make_inputs(1, 8)
    d = U.device_inputs(inp)
    perm = torch.tensor([3, 7, 0, 5, 1, 6, 2, 4], device="cuda")
    d2 = dict(d)
    d2["x"] = d["x"][perm].contiguous()
    a = _fwd(moe, d, 8)
    b = _fwd(moe, d2, 8)
    torch.cuda.synchronize()
    assert np.array_equal(_bits(b), _bits(a[perm]))


@pytest.mark.parametrize("H,I,E,k,M", [
    (96, 64, 3, 2, 5),        # tiny: one partial box, K tails in both projections
    (1056, 800, 16, 4, 9),    # H, I not multiples of the 512-element stage
    (256, 32, 1, 1, 3),       # a single expert: dense clamp-SwiGLU MLP
    (512, 256, 8, 8, 40),     # k == E: every token uses every expert, 16-wide tiles of 16, 16, 8
    (1056, 800, 16, 4, 40),   # 16-wide tiles (M*k >= 4E) with K tails and per-item scale rows
])
def test_ragged_shapes_against_oracle(moe, H, I, E, k, M):
    shape = gen.LayerShape("ragged", H, I, E, k, (M,))
    inp = gen.make_inputs(0, M, shape=shape, seed=H + I + E + k + M)
    d = U.device_inputs(inp)
    ids = torch.empty((M, k), dtype=torch.int32, device="cuda")
    ws = torch.empty(moe.moe_workspace_bytes(M, H, I, E, k), dtype=torch.uint8, device="cuda")
    out = moe.moe_mxfp4_forward_ex(d["x"], d["router_w"], d["w13_q"], d["w13_s"], d["w2_q"], d["w2_s"], k, ws,
                                   topk_ids_out=ids)
    torch.cuda.synchronize()
    r = U.oracle_forward(inp)
    assert np.array_equal(ids.cpu().numpy(), r["topk_ids"])
    U.check_out(U.bf16_tensor_to_f64(out), r["out64"], "ragged %s" % ((H, I, E, k, M),))


@pytest.mark.parametrize("H,I,E,k,M", [
    (1024, 512, 4, 2, 80),    # ~40 assignments per expert: every expert on the tensor-core path
    (512, 512, 4, 2, 600),    # ~300 per expert: two wide tiles per expert (192 + the rest)
    (512, 1024, 16, 4, 160),  # ~40 per expert with I > H
    (512, 512, 64, 4, 160),   # 3..19 per expert: mma.sync tiles and tensor-core tiles of N = 16 and 32
])
def test_wide_tiles_against_oracle(moe, H, I, E, k, M):
    # experts with U.WIDE_MIN_TOKENS or more assignments take the tcgen05 path (H, I multiples of 512)
    assert U.wide_path_on(M, H, I, E, k)
    shape = gen.LayerShape("wide", H, I, E, k, (M,))
    inp = gen.make_inputs(0, M, shape=shape, seed=7 * H + I + E + k + M)
    d = U.device_inputs(inp)
    ids = torch.empty((M, k), dtype=torch.int32, device="cuda")
    st = torch.full((1,), 123, dtype=torch.int32, device="cuda")
    ws = torch.empty(moe.moe_workspace_bytes(M, H, I, E, k), dtype=torch.uint8, device="cuda")
    out = moe.moe_mxfp4_forward_ex(d["x"], d["router_w"], d["w13_q"], d["w13_s"], d["w2_q"], d["w2_s"], k, ws,
                                   topk_ids_out=ids, status_out=st)
    torch.cuda.synchronize()
    assert int(st.item()) == moe.MOE_OK
    r = U.oracle_forward(inp)
    counts = np.bincount(r["topk_ids"].reshape(-1), minlength=E)
    assert counts.max() >= U.WIDE_MIN_TOKENS     # the case does reach the wide path
    assert np.array_equal(ids.cpu().numpy(), r["topk_ids"])
    U.check_out(U.bf16_tensor_to_f64(out), r["out64"], "wide %s" % ((H, I, E, k, M),))


def test_zero_tokens_is_a_no_op(moe):
    inp = gen.make_inputs(0, 2)
    d = U.device_inputs(inp)
    x0 = d["x"][:0]
    out = torch.empty((0, inp.shape.H), dtype=torch.bfloat16, device="cuda")
    r = moe.moe_mxfp4_forward(x0, d["router_w"], d["w13_q"], d["w13_s"], d["w2_q"], d["w2_s"], 4, out=out)
    assert r.shape == (0, inp.shape.H)


def test_status_out_reports_ok(moe):
    inp = gen.make_inputs(0, 2)
    d = U.device_inputs(inp)
    ws = torch.empty(moe.moe_workspace_bytes(2, 1024, 512, 16, 4), dtype=torch.uint8, device="cuda")
    st = torch.full((1,), -99, dtype=torch.int32, device="cuda")
    moe.moe_mxfp4_forward_ex(d["x"], d["router_w"], d["w13_q"], d["w13_s"], d["w2_q"], d["w2_s"], 4, ws,
                             status_out=st)
    torch.cuda.synchronize()
    assert int(st.item()) == moe.MOE_OK


def test_bounded_wait_gives_up_with_timeout_status(moe):
    # A wait that nothing completes runs out, reports MOE_ERR_TIMEOUT and ends the kernel; the
    # context stays usable and the next layer call reports MOE_OK with the same output as before.
    inp = gen.make_inputs(0, 2)
    d = U.device_inputs(inp)
    ws = torch.empty(moe.moe_workspace_bytes(2, 1024, 512, 16, 4), dtype=torch.uint8, device="cuda")
    before = moe.moe_mxfp4_forward_ex(d["x"], d["router_w"], d["w13_q"], d["w13_s"], d["w2_q"], d["w2_s"], 4, ws)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    moe.moe_selftest_wait_timeout(st)
    torch.cuda.synchronize()
    assert int(st.item()) == moe.MOE_ERR_TIMEOUT
    st2 = torch.full((1,), -99, dtype=torch.int32, device="cuda")
    after = moe.moe_mxfp4_forward_ex(d["x"], d["router_w"], d["w13_q"], d["w13_s"], d["w2_q"], d["w2_s"], 4, ws,
                                     status_out=st2)
    torch.cuda.synchronize()
    assert int(st2.item()) == moe.MOE_OK
    assert np.array_equal(_bits(before), _bits(after))


def test_generator_device_streams_match_host(moe):
    # the integer weight streams are bit-identical when generated on the device
    inp = gen.make_inputs(1, 2, weights="torch", device="cuda")
    for e in (0, 77, 127):
        q13, s13, q2, s2 = inp.expert_weights(e)
        assert np.array_equal(inp.w13_q[e].cpu().numpy(), q13)
        assert np.array_equal(inp.w13_s[e].cpu().numpy(), s13)
        assert np.array_equal(inp.w2_q[e].cpu().numpy(), q2)
        assert np.array_equal(inp.w2_s[e].cpu().numpy(), s2)
