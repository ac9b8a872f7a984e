"""moe_route_noalloc: the router for callers that cannot allocate device memory.

Such callers (an allocator that owns all device memory, a decode loop that must
not allocate between steps) use this entry point; its scratch lives in a fixed
device array inside the library.  It must give the same routing as moe_route.
This file is collected last so that a failure here comes after every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from moe_inputs import generator as gen
from tests import _gpu_util as U

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


@pytest.mark.parametrize("ci,M", [(2, 32), (1, 8), (4, 256)])
def test_noalloc_route_matches_route_on_consecutive_calls(ci, M):
    import decode_moe_layer_b200 as moe
    inp = gen.make_inputs(ci, M, weights="none")
    x = U.bits_to_bf16_tensor(inp.x)
    wr = torch.from_numpy(inp.router_w).cuda()
    bias = None if inp.router_bias is None else torch.from_numpy(inp.router_bias).cuda()
    k = inp.shape.k
    ref_ids, ref_w = moe.moe_route(x, wr, k, router_bias=bias)
    for _ in range(2):                       # two calls in a row share the static scratch
        ids, w = moe.moe_route_noalloc(x, wr, k, router_bias=bias)
        torch.cuda.synchronize()
        assert torch.equal(ids, ref_ids)
        assert float((w - ref_w).abs().max()) <= U.W_TOL


def test_noalloc_route_rejects_sizes_beyond_its_scratch():
    import decode_moe_layer_b200 as moe
    lib = moe.load()
    a = ctypes.c_void_p(0x1000)
    # 256 + 4096 * 512 * 4 bytes of logits exceed the 4 MiB array (M * k stays within limits)
    rc = lib.moe_route_noalloc(a, a, None, a, a, 4096, 7168, 512, 2, None)
    assert rc == moe.MOE_ERR_WORKSPACE
