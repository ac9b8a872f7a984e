"""The h tolerance of the GPU parity tests, checked on the CPU against an fp32 emulation of the
mma.sync kernel's arithmetic.

The emulation follows the kernel's order: per 32-element scale block the E2M1 x activation
products (exact in fp32) are summed in fp32, the block sum is scaled by its power-of-two E8M0
factor and added to one of eight fp32 K-slot accumulators (slot = block index mod 32, divided by
4), the slots are summed in slot order, and clamp-SwiGLU runs in fp32 before the bf16 rounding.
Like the GPU test it then reads h back from its binary16 storage (h * 2^10), which is exact only
for |h| >= 2^-27.  The derived bound (one bf16 ulp plus h's sensitivity to a worst-case fp32
accumulation error, plus the storage term) must accept it and must reject an h a few ulps off
where the bound is tight.  The flip rates match the GPU's (about 0.4% at H=2048, 6.5% at
H=7168), and nearly all flips are h values below 2^-27: the accumulation itself rarely flips a
rounding."""
import numpy as np
import pytest

import oracle
from moe_inputs import generator as gen
from tests import _gpu_util as U


def _emulate_h(x_bits, q, s):
    """fp32 emulation of one token through one expert's gate_up + clamp-SwiGLU (h as float64)."""
    xv = gen.bf16_bits_to_f64(x_bits).astype(np.float32)
    rows, K = q.shape[0], q.shape[1] * 2
    codes = np.empty((rows, K), np.float32)
    codes[:, 0::2] = U.E2M1[q & 15]
    codes[:, 1::2] = U.E2M1[q >> 4]
    prod = (codes * xv[None, :]).reshape(rows, K // 32, 32)          # exact products
    block = np.cumsum(prod, axis=2, dtype=np.float32)[:, :, -1]       # sequential fp32 block sums
    scale = (2.0 ** (s.astype(np.float64) - 127.0)).astype(np.float32)
    slots = np.zeros((8, rows), np.float32)
    for b in range(K // 32):
        slot = (b % 32) // 4
        slots[slot] = (slots[slot] + block[:, b] * scale[:, b]).astype(np.float32)
    acc = np.zeros(rows, np.float32)
    for sl in range(8):
        acc = (acc + slots[sl]).astype(np.float32)
    I = rows // 2
    g, u = acc[:I], acc[I:]
    a = np.minimum(g, np.float32(7.0))
    c = np.clip(u, np.float32(-7.0), np.float32(7.0))
    h32 = (a / (np.float32(1.0) + np.exp(-a)) * c).astype(np.float32)
    h = gen.bf16_bits_to_f64(gen._bf16_bits_rne(h32.astype(np.float64)))
    return (h * 1024.0).astype(np.float16).astype(np.float64) / 1024.0   # binary16 storage of h * 2^10


@pytest.mark.parametrize("ci,lo,hi", [(1, 0.001, 0.02), (2, 0.03, 0.12)])
def test_h_bound_accepts_fp32_kernel_order_and_rejects_real_errors(ci, lo, hi):
    inp = gen.make_inputs(ci, 2, weights="none")
    ids, _, _ = oracle.route(inp.x, inp.router_w, inp.router_bias, inp.shape.k)
    flips = total = big_flips = 0
    for t in range(inp.M):
        for j in range(4):   # four of each token's slots
            e = int(ids[t, j])
            q13, s13, _, _ = inp.expert_weights(e)
            g, u, ref_bits = oracle.expert_swiglu(inp.x[t], q13, s13)
            h = _emulate_h(inp.x[t], q13, s13)
            flips += U.check_h_bound(h, ref_bits, g, u, inp.x[t], q13, s13, "emulated c%d t=%d j=%d" % (ci, t, j))
            total += h.size
            ref = gen.bf16_bits_to_f64(ref_bits)
            big_flips += int(((h != ref) & (np.abs(ref) >= 2.0 ** -27)).sum())
            # a few ulps off where h does not depend on the accumulation (g and u both clamped)
            # must fail the bound
            tight = np.nonzero((g > 8.0) & (np.abs(u) > 8.0))[0]
            assert tight.size > 0
            bad = h.copy()
            bad[tight[0]] += 4 * U.bf16_ulp(np.abs(ref[tight[0]]))
            with pytest.raises(AssertionError):
                U.check_h_bound(bad, ref_bits, g, u, inp.x[t], q13, s13, "planted")
    # the GPU's flip rates, almost all from the binary16 storage of h below 2^-27
    assert lo * total <= flips <= hi * total, (flips, total)
    assert big_flips <= 0.001 * total, (big_flips, total)
