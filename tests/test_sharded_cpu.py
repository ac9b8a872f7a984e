"""The I-sharded layer's host logic on the CPU.

Weight slicing (decode_moe_layer_b200.sharded.shard_weights) and the exchange of the ranks'
shares (gather_partials, two gloo ranks) are the product's own code; the oracle stands in for
each rank's GPU share (its fp64 out64 of the sliced layer is the unrounded weighted top-k sum
that moe_mxfp4_forward_partial returns in fp32).  The rank-order sum of the shares must equal the
oracle's unsplit layer, because every intermediate element h_i is computed from the same full-H
dot products in either case and the down projection's K sum only regroups."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from decode_moe_layer_b200 import sharded
from moe_inputs import generator as gen

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_share(inp, rank, world):
    sl = sharded.shard_weights(inp.w13_q, inp.w13_s, inp.w2_q, inp.w2_s, rank, world)
    return oracle.forward(inp.x, inp.router_w, inp.router_bias, *sl, inp.shape.k)


def test_shard_weights_partitions_every_row_and_block_once():
    inp = gen.make_inputs(0, 2)
    E, I2, Hh = inp.w13_q.shape
    I, world = I2 // 2, 4
    parts = [sharded.shard_weights(inp.w13_q, inp.w13_s, inp.w2_q, inp.w2_s, r, world) for r in range(world)]
    n = I // world
    for q13, s13, q2, s2 in parts:
        assert q13.shape == (E, 2 * n, Hh) and s13.shape == (E, 2 * n, inp.w13_s.shape[2])
        assert q2.shape == (E, inp.w2_q.shape[1], n // 2) and s2.shape == (E, inp.w2_s.shape[1], n // 32)
        assert all(a.flags["C_CONTIGUOUS"] for a in (q13, s13, q2, s2))
    # gate slices in rank order rebuild the gate rows, up slices the up rows, w2 slices the K range
    np.testing.assert_array_equal(np.concatenate([p[0][:, :n] for p in parts], axis=1), inp.w13_q[:, :I])
    np.testing.assert_array_equal(np.concatenate([p[0][:, n:] for p in parts], axis=1), inp.w13_q[:, I:])
    np.testing.assert_array_equal(np.concatenate([p[1][:, n:] for p in parts], axis=1), inp.w13_s[:, I:])
    np.testing.assert_array_equal(np.concatenate([p[2] for p in parts], axis=2), inp.w2_q)
    np.testing.assert_array_equal(np.concatenate([p[3] for p in parts], axis=2), inp.w2_s)
    # torch tensors slice the same way
    t = sharded.shard_weights(*(torch.from_numpy(a) for a in (inp.w13_q, inp.w13_s, inp.w2_q, inp.w2_s)), 1, world)
    for a, b in zip(t, parts[1]):
        np.testing.assert_array_equal(a.numpy(), b)
    # one rank keeps everything
    for a, b in zip(sharded.shard_weights(inp.w13_q, inp.w13_s, inp.w2_q, inp.w2_s, 0, 1),
                    (inp.w13_q, inp.w13_s, inp.w2_q, inp.w2_s)):
        np.testing.assert_array_equal(a, b)


def test_shard_bounds_refuses_splits_inside_a_scale_block():
    assert sharded.shard_bounds(512, 3, 4) == (384, 512)
    with pytest.raises(ValueError):
        sharded.shard_bounds(512, 0, 32)     # 16 rows: half a scale block
    with pytest.raises(ValueError):
        sharded.shard_bounds(768, 0, 5)      # not a whole split
    with pytest.raises(ValueError):
        sharded.shard_bounds(512, 4, 4)


def test_four_oracle_shares_sum_to_the_unsplit_layer():
    inp = gen.make_inputs(0, 2)
    full = oracle.forward(inp.x, inp.router_w, inp.router_bias, inp.w13_q, inp.w13_s, inp.w2_q, inp.w2_s,
                          inp.shape.k)
    world = 4
    shares = [_oracle_share(inp, r, world) for r in range(world)]
    total = np.zeros_like(full["out64"])
    for s in shares:
        np.testing.assert_array_equal(s["topk_ids"], full["topk_ids"])
        total += s["out64"]
    np.testing.assert_allclose(total, full["out64"], rtol=0, atol=1e-12 * np.abs(full["out64"]).max())
    # each share's h is the matching column range of the unsplit layer's h
    n = inp.shape.I // world
    for r, s in enumerate(shares):
        np.testing.assert_array_equal(s["h"], full["h"][:, r * n:(r + 1) * n])


def _rank_main(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        inp = gen.make_inputs(0, 2)
        mine = _oracle_share(inp, rank, world)
        stack = sharded.gather_partials(torch.from_numpy(mine["out64"]))
        total = stack[0].clone()
        for g in range(1, stack.shape[0]):   # rank order, the order moe_reduce_partials uses
            total += stack[g]
        q.put((rank, total.numpy(), stack.numpy(), mine["out64"]))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_exchange_shares_in_rank_order():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    for _ in range(world):
        rank, total, stack, own = q.get(timeout=180)
        got[rank] = (total, stack, own)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # slot g of the gathered stack is rank g's own share, on both ranks
    for r in range(world):
        for g in range(world):
            np.testing.assert_array_equal(got[r][1][g], got[g][2])
    # both ranks hold the same bits, equal to the unsplit layer
    np.testing.assert_array_equal(got[0][0], got[1][0])
    inp = gen.make_inputs(0, 2)
    full = oracle.forward(inp.x, inp.router_w, inp.router_bias, inp.w13_q, inp.w13_s, inp.w2_q, inp.w2_s,
                          inp.shape.k)
    np.testing.assert_allclose(got[0][0], full["out64"], rtol=0, atol=1e-12 * np.abs(full["out64"]).max())
