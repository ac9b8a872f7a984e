"""The bench's per-launch accounting follows the library's launch plan (CPU only).

bench.py attributes algorithmic bytes to the launches a call makes (the tensor-core path, the fused
down + combine launch of the smallest calls) with rules of its own; here they are checked against
the library's host planner through moe_forward_launches, which needs no GPU."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

moe = pytest.importorskip("decode_moe_layer_b200")
import bench  # noqa: E402
from moe_inputs import generator as gen  # noqa: E402

SHAPES = list(gen.CONFIGS) + [
    gen.LayerShape("small_e", 512, 512, 8, 8, (1,)),
    gen.LayerShape("k1", 256, 256, 8, 1, (1,)),
    gen.LayerShape("ragged", 1056, 800, 16, 4, (1,)),
    gen.LayerShape("i1024", 1024, 1024, 32, 4, (1,)),
]


def _fused_select(M, E, k):
    # top-k and the permutation as one kernel: M <= 64, M*k <= 1024, M*E <= 16384 (moe_internal.h)
    return M <= 64 and M * k <= 1024 and M * E <= 16384


@pytest.mark.parametrize("shape", SHAPES, ids=[s.name for s in SHAPES])
def test_launch_classes_match_the_library(shape):
    for M in list(range(1, 41)) + [64, 96, 256, 512, 1024]:
        if M * shape.k > 16384:
            continue
        want = ((5 if _fused_select(M, shape.E, shape.k) else 6) + (5 if bench.wide_on(shape, M) else 0)
                - (1 if bench.down_fused(shape, M) else 0))
        got = moe.moe_forward_launches(M, shape.H, shape.I, shape.E, shape.k)
        assert got == want, (shape.name, M, got, want)


def test_fused_down_serves_the_smallest_workload_calls():
    tiny, decode = gen.CONFIGS[0], gen.CONFIGS[1]
    assert bench.down_fused(tiny, 1) and bench.down_fused(tiny, 2) and not bench.down_fused(tiny, 3)
    assert bench.down_fused(decode, 1) and not bench.down_fused(decode, 2)
    assert not any(bench.down_fused(c, M) for c in gen.CONFIGS[2:] for M in c.Ms)
