"""The layer split over G GPUs along the expert intermediate dimension I ("I-sharding").

Every rank keeps every expert, but only I/G of its intermediate rows: gate rows and up rows
[r*I/G, (r+1)*I/G) of w13 and the same K range of w2.  That slice is itself a layer of
intermediate size I/G, so one rank's call is the single-GPU path unchanged except for its
last step, which keeps the weighted top-k sum in fp32 (moe_mxfp4_forward_partial).  The ranks
then all-gather their [M,H] fp32 shares in rank order over the process group (NCCL over
NVLink on GPUs) and each sums them in that fixed order and rounds once to bf16
(moe_reduce_partials), so all ranks hold the same bits.

Why this split and not expert parallelism: the pages' one multi-GPU data point ("The Systematic
Optimization Campaign", chunk 8.0) has 8-way expert parallelism slower than a single GPU at low
concurrency and failing under load; an I-split keeps every rank's weight stream the same size
whatever the routing skew, and exchanges only M*H*4 bytes per rank, against the layer's
gigabytes of weights.

Routing is computed in full on every rank from the replicated x and router weights, which gives
every rank the same ids and weights bit for bit (the router kernels are deterministic).
"""
from __future__ import annotations

import numpy as np
import torch
import torch.distributed as dist

from . import _lib


def shard_bounds(I: int, rank: int, world: int):
    """[lo, hi) of the intermediate rows rank `rank` of `world` keeps."""
    if world <= 0 or not 0 <= rank < world:
        raise ValueError("rank %d of %d" % (rank, world))
    if I % world != 0 or (I // world) % 32 != 0:
        raise ValueError("I=%d does not split into %d slices of whole 32-element scale blocks" % (I, world))
    n = I // world
    return rank * n, (rank + 1) * n


def shard_weights(w13_q, w13_s, w2_q, w2_s, rank: int, world: int):
    """This rank's (w13_q, w13_s, w2_q, w2_s): a layer of intermediate size I/world.

    w13 [E, 2I, ...] holds the gate rows 0..I-1 then the up rows I..2I-1; the slice keeps gate rows
    [lo, hi) followed by up rows [I+lo, I+hi).  w2 [E, H, I/2] (scales [E, H, I/32]) keeps the K range
    [lo, hi): packed bytes [lo/2, hi/2), scale bytes [lo/32, hi/32).  Accepts numpy arrays or torch
    tensors (any device) and returns contiguous copies of the same kind.
    """
    I = w13_q.shape[1] // 2
    lo, hi = shard_bounds(I, rank, world)
    if isinstance(w13_q, torch.Tensor):
        cat, contig = (lambda a, b: torch.cat([a, b], dim=1)), (lambda a: a.contiguous())
    else:
        cat, contig = (lambda a, b: np.concatenate([a, b], axis=1)), np.ascontiguousarray
    q13 = cat(w13_q[:, lo:hi], w13_q[:, I + lo:I + hi])
    s13 = cat(w13_s[:, lo:hi], w13_s[:, I + lo:I + hi])
    q2 = contig(w2_q[:, :, lo // 2:hi // 2])
    s2 = contig(w2_s[:, :, lo // 32:hi // 32])
    return q13, s13, q2, s2


def gather_partials(partial, group=None):
    """[G, M, H] stack of every rank's [M, H] share, in rank order (one all-gather)."""
    world = dist.get_world_size(group)
    stack = partial.new_empty((world,) + tuple(partial.shape))
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(stack, partial.contiguous(), group=group)
    else:
        dist.all_gather(list(stack.unbind(0)), partial.contiguous(), group=group)
    return stack


class IShardedLayer:
    """One rank of the I-sharded layer.  Holds this rank's weight slices on its GPU and a
    workspace; forward() runs this rank's share, the exchange and the fixed-order reduction."""

    def __init__(self, w13_q, w13_s, w2_q, w2_s, k: int, group=None, device=None):
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        self.k = k
        dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        sl = shard_weights(w13_q, w13_s, w2_q, w2_s, self.rank, self.world)
        self.w13_q, self.w13_s, self.w2_q, self.w2_s = (
            (t if isinstance(t, torch.Tensor) else torch.from_numpy(t)).to(dev) for t in sl)
        self.E, self.H = self.w2_q.shape[0], self.w2_q.shape[1]
        self.I_shard = self.w13_q.shape[1] // 2
        self._ws = None

    def workspace(self, M: int):
        need = _lib.moe_workspace_bytes(M, self.H, self.I_shard, self.E, self.k)
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty(max(need, 256), dtype=torch.uint8, device=self.w13_q.device)
        return self._ws

    def partial(self, x, router_w, router_bias=None, partial_out=None, topk_ids_out=None, status_out=None):
        """This rank's fp32 [M, H] share (on the current stream)."""
        return _lib.moe_mxfp4_forward_partial(x, router_w, self.w13_q, self.w13_s, self.w2_q, self.w2_s, self.k,
                                              self.workspace(x.shape[0]), router_bias=router_bias,
                                              partial_out=partial_out, topk_ids_out=topk_ids_out,
                                              status_out=status_out)

    def forward(self, x, router_w, router_bias=None, out=None, status_out=None):
        """out [M, H] bf16, the same bits on every rank."""
        part = self.partial(x, router_w, router_bias=router_bias, status_out=status_out)
        return _lib.moe_reduce_partials(gather_partials(part, self.group), out=out)
