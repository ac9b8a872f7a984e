"""Shared helpers for the GPU parity tests: device upload of the seeded inputs,
calls into the oracle for the same inputs, and the tolerance checks.

Tolerances (derivations in the design notes):
  * routing ids, expert offsets, sorted ids, inverse positions: bit-exact;
  * routing weights: |w - w_oracle| <= 1e-5 (fp32 logits and softmax vs fp64);
  * h: within one bf16 ulp of the oracle's bf16 value plus h's sensitivity to a
    worst-case fp32 accumulation error (check_h_bound), flips counted;
  * out: relative L2 error <= 5e-3 and max abs error <= 2e-2 * rms, both against
    the oracle's fp64 out64.
"""
from __future__ import annotations

import os

import numpy as np
import torch

import oracle
from moe_inputs import generator as gen

W_TOL = 1e-5
REL_L2_TOL = 5e-3
MAX_ABS_RMS_TOL = 2e-2


def bits_to_bf16_tensor(bits: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device).view(torch.bfloat16)


def bf16_tensor_to_f64(t: torch.Tensor) -> np.ndarray:
    return gen.bf16_bits_to_f64(t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16))


def device_inputs(inp: gen.MoEInputs, device="cuda"):
    def dev(a):
        if isinstance(a, torch.Tensor):
            return a.to(device).contiguous()
        return torch.from_numpy(np.ascontiguousarray(a)).to(device)

    d = {
        "x": bits_to_bf16_tensor(inp.x, device),
        "router_w": torch.from_numpy(inp.router_w).to(device),
        "router_bias": None if inp.router_bias is None else torch.from_numpy(inp.router_bias).to(device),
        "w13_q": dev(inp.w13_q), "w13_s": dev(inp.w13_s), "w2_q": dev(inp.w2_q), "w2_s": dev(inp.w2_s),
    }
    return d


def _expert_host(inp: gen.MoEInputs, e: int):
    """One expert's weights on the host.  Weights generated on the device by the generator's torch
    streams are copied back (test_generator_device_streams_match_host checks that those streams
    equal the host ones bit for bit); host arrays are used as they are."""
    if isinstance(inp.w13_q, np.ndarray):
        return inp.w13_q[e], inp.w13_s[e], inp.w2_q[e], inp.w2_s[e]
    return tuple(a[e].cpu().numpy() for a in (inp.w13_q, inp.w13_s, inp.w2_q, inp.w2_s))


def oracle_forward(inp: gen.MoEInputs, tokens=None):
    """Oracle layer output for `tokens` (all when None), passing only the experts they touch."""
    k = inp.shape.k
    if isinstance(inp.w13_q, np.ndarray):
        return oracle.forward(inp.x, inp.router_w, inp.router_bias, inp.w13_q, inp.w13_s, inp.w2_q, inp.w2_s, k,
                              tokens=tokens, I=inp.shape.I)
    ids, _, _ = oracle.route(inp.x, inp.router_w, inp.router_bias, k)
    toks = range(inp.M) if tokens is None else tokens
    need = sorted(set(int(e) for t in toks for e in ids[t]))
    ex = {e: _expert_host(inp, e) for e in need}
    return oracle.forward(inp.x, inp.router_w, inp.router_bias,
                          {e: v[0] for e, v in ex.items()}, {e: v[1] for e, v in ex.items()},
                          {e: v[2] for e, v in ex.items()}, {e: v[3] for e, v in ex.items()},
                          k, tokens=tokens, I=inp.shape.I)


def check_out(gpu_out: np.ndarray, ref64: np.ndarray, what=""):
    """gpu_out: float64 values of the bf16 output rows; ref64: the oracle's fp64 rows."""
    err = gpu_out - ref64
    rms = float(np.sqrt(np.mean(ref64 ** 2)))
    rel_l2 = float(np.linalg.norm(err) / max(np.linalg.norm(ref64), 1e-300))
    max_abs = float(np.abs(err).max())
    assert np.all(np.isfinite(gpu_out)), what + ": non-finite output"
    assert rel_l2 <= REL_L2_TOL, "%s: rel L2 %.3e > %.1e" % (what, rel_l2, REL_L2_TOL)
    assert max_abs <= MAX_ABS_RMS_TOL * rms, "%s: max abs %.3e > %.1e * rms %.3e" % (what, max_abs,
                                                                                    MAX_ABS_RMS_TOL, rms)
    return rel_l2, max_abs / rms


def check_out_heavy_tailed(gpu_out: np.ndarray, ref64: np.ndarray, what=""):
    """check_out's relative L2 bar, and per element the max-abs bar plus the element's own bf16
    rounding (2^-9 |ref|, doubled for the fp32 accumulation): for outputs whose largest elements sit
    far above their rms, a single correctly rounded element can exceed 2e-2 * rms by itself."""
    err = np.abs(gpu_out - ref64)
    rms = float(np.sqrt(np.mean(ref64 ** 2)))
    rel_l2 = float(np.linalg.norm(gpu_out - ref64) / max(np.linalg.norm(ref64), 1e-300))
    assert np.all(np.isfinite(gpu_out)), what + ": non-finite output"
    assert rel_l2 <= REL_L2_TOL, "%s: rel L2 %.3e > %.1e" % (what, rel_l2, REL_L2_TOL)
    bound = MAX_ABS_RMS_TOL * rms + 2.0 ** -8 * np.abs(ref64)
    worst = float((err / bound).max())
    assert worst <= 1.0, "%s: an element exceeds 2e-2 * rms + 2^-8 |ref| by %.2fx" % (what, worst)
    return rel_l2, worst


def bf16_ulp(v: np.ndarray) -> np.ndarray:
    a = np.maximum(np.abs(v), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(a)) - 7)


FLIP_LOG = []


def _e2m1_table():
    vals = {}
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "e2m1_ocp_mx_v1.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                c, v = line.split()
                vals[int(c)] = float(v)
    return np.array([vals[c] for c in range(16)])


E2M1 = _e2m1_table()


def decode_mx(q: np.ndarray, s: np.ndarray) -> np.ndarray:
    """Dequantise an MXFP4 matrix [rows, K/2] + [rows, K/32] with the OCP table fixture."""
    vals = np.empty(q.shape[:-1] + (q.shape[-1] * 2,))
    vals[..., 0::2] = E2M1[q & 15]
    vals[..., 1::2] = E2M1[q >> 4]
    return vals * np.repeat(2.0 ** (s.astype(np.float64) - 127.0), 32, axis=-1)


def _silu(z):
    return z / (1.0 + np.exp(-z))


def _dsilu(z):
    sg = 1.0 / (1.0 + np.exp(-z))
    return sg * (1.0 + z * (1.0 - sg))


def check_h_bound(gpu_h, ref_bits, g, u, x_row_bits, w13_q_e, w13_s_e, what=""):
    """h within one bf16 ulp of the oracle plus its sensitivity to the fp32 accumulation error.

    The GPU sums each gate/up dot product in fp32 (exact bf16 products, at most ~100
    sequential fp32 roundings per output); its error is bounded by
    eps = 2^-17 * sum_k |w_k x_k| (a worst-case bound, not a statistical one).  h
    moves by at most |dh/dg| eps_g + |dh/du| eps_u, and the GPU rounds h to bf16 once,
    as the oracle does.  Flips are recorded in FLIP_LOG."""
    ref = gen.bf16_bits_to_f64(ref_bits)
    I = ref.shape[0]
    W = decode_mx(w13_q_e, w13_s_e)
    ax = np.abs(gen.bf16_bits_to_f64(x_row_bits))
    S = np.abs(W) @ ax
    eps_g, eps_u = 2.0 ** -17 * S[:I], 2.0 ** -17 * S[I:]
    a = np.minimum(g, 7.0)
    c = np.clip(u, -7.0, 7.0)
    dg = np.where(g < 7.0 + eps_g, np.abs(_dsilu(a) * c), 0.0)
    du = np.where(np.abs(u) < 7.0 + eps_u, np.abs(_silu(a)), 0.0)
    tol = bf16_ulp(np.abs(ref)) + dg * eps_g + du * eps_u
    diff = np.abs(gpu_h - ref)
    bad = diff > tol
    assert not bad.any(), "%s: %d elements beyond the derived bound (worst excess %.3e at h=%.3e)" % (
        what, int(bad.sum()), float((diff - tol).max()), float(ref[np.argmax(diff - tol)]))
    flips = int((diff > 0).sum())
    FLIP_LOG.append((what, flips, diff.size))
    return flips


# The library's split of an expert's assignments into tiles (moe_internal.h): mma.sync tiles of
# 16 once the experts average 6 or more assignments (else 8); when H and I are multiples of 512 and
# the call is wide enough, tensor-core tiles for an expert with WIDE_MIN_TOKENS or more: one tile
# up to WIDE_SMALL_MAX assignments, else tiles of up to WIDE_TOKENS.
WIDE_MIN_TOKENS = 5
WIDE_SMALL_MAX = 64
WIDE_TOKENS = 192


def wide_path_on(M, H, I, E, k):
    return M >= WIDE_MIN_TOKENS and H % 512 == 0 and I % 512 == 0 and 2 * M * k >= WIDE_MIN_TOKENS * E


def sample_tokens(ids: np.ndarray, E: int, H: int, I: int, n_min=64, cap=112, seed=0):
    """Tokens to compare at full size: all when M <= n_min; else tokens that put an assignment on
    every slot position and every fill count of the mma.sync tiles, the first and last assignment
    of the tensor-core tiles (in random order, up to `cap` tokens in all), then random tokens up
    to n_min.  Returns (sorted token list, description)."""
    M, k = ids.shape
    if M <= n_min:
        return list(range(M)), "all %d tokens" % M
    rng = np.random.default_rng(seed)
    off, srt, _ = oracle.permute(ids, E)
    counts = np.diff(off)
    W = 16 if M * k >= 6 * E else 8
    wide_on = wide_path_on(M, H, I, E, k)
    want, slots, fills, wide_ends = set(), set(), set(), []
    for e in range(E):
        c = int(counts[e])
        if c == 0:
            continue
        p = int(off[e])
        if wide_on and c >= WIDE_MIN_TOKENS:
            step = c if c <= WIDE_SMALL_MAX else WIDE_TOKENS
            for t0 in range(0, c, step):
                n = min(step, c - t0)
                wide_ends.append((int(srt[p + t0]) // k, int(srt[p + t0 + n - 1]) // k))
            continue
        for t0 in range(0, c, W):
            n = min(W, c - t0)
            if n not in fills:
                fills.add(n)
                want.add(int(srt[p + t0 + n - 1]) // k)
            for sl in range(n):
                if sl not in slots:
                    slots.add(sl)
                    want.add(int(srt[p + t0 + sl]) // k)
    n_wide = len(wide_ends)
    for i in rng.permutation(n_wide):
        if len(want) + 2 > cap:
            break
        want.update(wide_ends[i])
    covered = sum(1 for a, b in wide_ends if a in want and b in want)
    for t in rng.permutation(M):
        if len(want) >= n_min:
            break
        want.add(int(t))
    desc = ("%d tokens: mma.sync slots %s, fills %s; ends of %d of %d tensor-core tiles"
            % (len(want), sorted(slots), sorted(fills), covered, n_wide))
    return sorted(want), desc
