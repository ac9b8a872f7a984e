"""GPU parity of the I-sharded layer, its G ranks run one after another on one GPU.

Each rank's share comes from moe_mxfp4_forward_partial on the weight slices shard_weights cuts
(the same call each rank of a multi-GPU run makes); the shares are stacked in rank order, as the
all-gather leaves them, and moe_reduce_partials sums them in that fixed order.  Nothing here waits
on another rank: the exchange itself is covered by the gloo test on the CPU."""
import numpy as np
import oracle
import pytest
import torch

from decode_moe_layer_b200 import sharded
from moe_inputs import generator as gen
from tests import _gpu_util as U

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


@pytest.fixture(scope="module")
def moe():
    import decode_moe_layer_b200 as m
    return m


def _run_shards(moe, d, inp, world):
    M, H, E, k = inp.M, inp.shape.H, inp.shape.E, inp.shape.k
    I_shard = inp.shape.I // world
    parts, ids_all = [], []
    for r in range(world):
        q13, s13, q2, s2 = sharded.shard_weights(d["w13_q"], d["w13_s"], d["w2_q"], d["w2_s"], r, world)
        ws = torch.empty(moe.moe_workspace_bytes(M, H, I_shard, E, k), dtype=torch.uint8, device="cuda")
        ids = torch.empty((M, k), dtype=torch.int32, device="cuda")
        st = torch.full((1,), 123, dtype=torch.int32, device="cuda")
        p = moe.moe_mxfp4_forward_partial(d["x"], d["router_w"], q13, s13, q2, s2, k, ws,
                                          router_bias=d["router_bias"], topk_ids_out=ids, status_out=st)
        torch.cuda.synchronize()
        assert int(st.item()) == moe.MOE_OK
        parts.append(p)
        ids_all.append(ids.cpu().numpy())
    return torch.stack(parts), ids_all


# (shape, M, G): the tiny and decode-width layers on mma.sync tiles, and a layer whose I/G = 512
# slices keep the tensor-core tiles (M*k/E = 40 assignments per expert)
CASES = [
    ("tiny", gen.CONFIGS[0], 2, 2),
    ("decode", gen.CONFIGS[1], 8, 2),
    ("decode", gen.CONFIGS[1], 96, 4),
    ("tc", gen.LayerShape("tc_h1024_i1024_e4_k2", 1024, 1024, 4, 2, (80,)), 80, 2),
]


@pytest.mark.parametrize("name,shape,M,world", CASES, ids=["%s-M%d-G%d" % (c[0], c[2], c[3]) for c in CASES])
def test_sharded_layer_matches_oracle(moe, name, shape, M, world):
    inp = gen.make_inputs(0, M, shape=shape, seed=4242 + M)
    d = U.device_inputs(inp)
    if name == "tc":
        assert U.wide_path_on(M, shape.H, shape.I // world, shape.E, shape.k)
    stack, ids_all = _run_shards(moe, d, inp, world)
    out = moe.moe_reduce_partials(stack)
    torch.cuda.synchronize()
    r = U.oracle_forward(inp)
    for ids in ids_all:   # every rank routes identically
        assert np.array_equal(ids, r["topk_ids"])
    U.check_out(U.bf16_tensor_to_f64(out), r["out64"], "sharded %s M=%d G=%d" % (name, M, world))
    # each share alone is the oracle's share of its slice (fp32 vs fp64, before any rounding)
    for g in range(world):
        sl = sharded.shard_weights(inp.w13_q, inp.w13_s, inp.w2_q, inp.w2_s, g, world)
        rg = oracle.forward(inp.x, inp.router_w, inp.router_bias, *sl, shape.k)
        ref = rg["out64"]
        got = stack[g].cpu().numpy().astype(np.float64)
        rel = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300)
        assert rel <= U.REL_L2_TOL, (g, rel)


def test_one_shard_reduces_to_the_unsplit_call(moe):
    inp = gen.make_inputs(1, 8)
    d = U.device_inputs(inp)
    k = inp.shape.k
    ws = torch.empty(moe.moe_workspace_bytes(8, inp.shape.H, inp.shape.I, inp.shape.E, k), dtype=torch.uint8,
                     device="cuda")
    full = moe.moe_mxfp4_forward_ex(d["x"], d["router_w"], d["w13_q"], d["w13_s"], d["w2_q"], d["w2_s"], k, ws,
                                    router_bias=d["router_bias"])
    stack, _ = _run_shards(moe, d, inp, 1)
    out = moe.moe_reduce_partials(stack)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), full.view(torch.int16))


@pytest.mark.parametrize("G,M,H", [(1, 3, 64), (3, 5, 7168), (8, 2, 2048)])
def test_reduce_partials_bit_exact(moe, G, M, H):
    rng = np.random.default_rng(G * 1000 + M)
    p = (rng.standard_normal((G, M, H)) * np.exp2(rng.integers(-30, 30, (G, M, H)))).astype(np.float32)
    p[0, 0, :4] = [1.0, -1.0, 2.0 ** -140, 3.0e38]
    out = moe.moe_reduce_partials(torch.from_numpy(p).cuda())
    torch.cuda.synchronize()
    acc = p[0].copy()
    for g in range(1, G):
        acc = (acc + p[g]).astype(np.float32)   # fp32 adds in rank order
    want = gen._bf16_bits_rne(acc.astype(np.float64))
    got = out.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got, want)
