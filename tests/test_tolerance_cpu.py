"""The h tolerance of the GPU parity tests, checked on the CPU against an fp32 emulation of the
mma.sync kernel's arithmetic.

The emulation follows the kernel's order: each 32-element scale block feeds two MMAs of 16 exact
products of the E2M1 values and the bf16 activations (K = 0,1,4,5 and 2,3,6,7 mod 8 inside every
group of 8, the decode's pairing), the second adding to the first's fp32 result; the block's fp32
partial times its power-of-two E8M0 factor joins one of eight fp32 K-slot accumulators (slot =
block index mod 32, divided by 4); the slots are summed in slot order, and clamp-SwiGLU runs in
fp32 before the one bf16 rounding of h.  The derived bound (one bf16 ulp plus h's sensitivity to
a worst-case fp32 accumulation error) must accept it and must reject an h a few ulps off where
the bound is tight.  Only the fp32 accumulation can flip a rounding of h against the fp64 oracle,
and it rarely does."""
import numpy as np
import pytest

import oracle
from moe_inputs import generator as gen
from tests import _gpu_util as U


def _emulate_h(x_bits, q, s):
    """fp32 emulation of one token through one expert's gate_up + clamp-SwiGLU (h as float64)."""
    xv = gen.bf16_bits_to_f64(x_bits)
    rows, K = q.shape[0], q.shape[1] * 2
    codes = np.empty((rows, K))
    codes[:, 0::2] = U.E2M1[q & 15]
    codes[:, 1::2] = U.E2M1[q >> 4]
    prod = (codes * xv[None, :]).reshape(rows, K // 32, 32)               # exact products
    lane = np.arange(32) % 8
    first = np.isin(lane, (0, 1, 4, 5))
    m1 = prod[:, :, first].sum(axis=2).astype(np.float32)
    block = (m1.astype(np.float64) + prod[:, :, ~first].sum(axis=2)).astype(np.float32)
    scale = (2.0 ** (s.astype(np.float64) - 127.0)).astype(np.float32)
    slots = np.zeros((8, rows), np.float32)
    for b in range(K // 32):
        slot = (b % 32) // 4
        slots[slot] = (slots[slot].astype(np.float64) + block[:, b].astype(np.float64) * scale[:, b]).astype(np.float32)
    acc = np.zeros(rows, np.float32)
    for sl in range(8):
        acc = (acc + slots[sl]).astype(np.float32)
    I = rows // 2
    g, u = acc[:I], acc[I:]
    a = np.minimum(g, np.float32(7.0))
    c = np.clip(u, np.float32(-7.0), np.float32(7.0))
    h32 = (a / (np.float32(1.0) + np.exp(-a)) * c).astype(np.float32)
    return gen.bf16_bits_to_f64(gen._bf16_bits_rne(h32.astype(np.float64)))


@pytest.mark.parametrize("ci", [1, 2])
def test_h_bound_accepts_fp32_kernel_order_and_rejects_real_errors(ci):
    inp = gen.make_inputs(ci, 2, weights="none")
    ids, _, _ = oracle.route(inp.x, inp.router_w, inp.router_bias, inp.shape.k)
    flips = total = 0
    for t in range(inp.M):
        for j in range(4):   # four of each token's slots
            e = int(ids[t, j])
            q13, s13, _, _ = inp.expert_weights(e)
            g, u, ref_bits = oracle.expert_swiglu(inp.x[t], q13, s13)
            h = _emulate_h(inp.x[t], q13, s13)
            flips += U.check_h_bound(h, ref_bits, g, u, inp.x[t], q13, s13, "emulated c%d t=%d j=%d" % (ci, t, j))
            total += h.size
            ref = gen.bf16_bits_to_f64(ref_bits)
            # a few ulps off where h does not depend on the accumulation (g and u both clamped)
            # must fail the bound
            tight = np.nonzero((g > 8.0) & (np.abs(u) > 8.0))[0]
            assert tight.size > 0
            bad = h.copy()
            bad[tight[0]] += 4 * U.bf16_ulp(np.abs(ref[tight[0]]))
            with pytest.raises(AssertionError):
                U.check_h_bound(bad, ref_bits, g, u, inp.x[t], q13, s13, "planted")
    # fp32 accumulation flips very few bf16 roundings of h
    assert flips <= 0.001 * total, (flips, total)
