"""Counter-based synthetic input generator for the routed MXFP4 MoE layer.

Every value is a pure function of (seed, stream tag, index), so any slice -- one
expert's weights, one token's activations -- can be regenerated on its own, on
the host (numpy) or on a device (torch), with identical bits for the integer
streams (weight nibbles and scale bytes).

Random source: the splitmix64 output function (G. Steele, D. Lea, C. Flood,
"Fast splittable pseudorandom number generators", OOPSLA 2014) applied to the
counter sequence base + (i+1)*0x9E3779B97F4A7C15.  Normals come from the
Box-Muller transform of two uniforms.

Workload shapes follow the decode MoE layers the pages profile: the Qwen3-MoE
class layer of "row/QUANT-CT-MXFP4-C8-DIFF" (vllm.cpp PR #52, per-step diff at
c8, M=8) and the DeepSeek class routed layer of "MTP1 Post-Portfolio Eager-Cycle
Profile" (table "Post-Portfolio Device Attribution", compact routed MXFP4 GEMM).
The value distributions are this library's synthetic recipe: x ~ N(0,1) rounded
to bf16, router weights ~ N(0, 1/H) fp32, every E2M1 nibble uniform over its 16
codes, every E8M0 scale byte uniform over {120..124}.

The only arithmetic on the layer's data in this module is the precondition check
`margin_ok`: it computes fp64 router logits to guarantee that the k+1 largest
logits of every token are separated by at least 1e-4, so that the expert choice
is decided well above fp32 rounding; tokens that miss the margin are redrawn.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence

import numpy as np

GAMMA = 0x9E3779B97F4A7C15
_MIX1 = 0xBF58476D1CE4E5B9
_MIX2 = 0x94D049BB133111EB
_MASK64 = (1 << 64) - 1

MARGIN = 1e-4
SCALE_LO, SCALE_N = 120, 5          # E8M0 scale bytes uniform over {120..124}

# stream tags (arbitrary distinct 32-bit constants)
_TAG_X = 0x78000000
_TAG_WR = 0x57520000
_TAG_W13Q = 0x31335100
_TAG_W13S = 0x31335300
_TAG_W2Q = 0x00325100
_TAG_W2S = 0x00325300


# --------------------------------------------------------------------------- shapes

@dataclasses.dataclass(frozen=True)
class LayerShape:
    name: str
    H: int
    I: int
    E: int
    k: int
    Ms: tuple
    skew_bias: bool = False

    @property
    def default_M(self) -> int:
        return self.Ms[-1]


# The five workloads: tiny layer; decode-width Qwen3-MoE-like layer; DeepSeek-V3
# class routed layer at decode and at wider batches; skewed routing stress.
CONFIGS = (
    LayerShape("tiny_h1024_i512_e16_k4", 1024, 512, 16, 4, (2,)),
    LayerShape("decode_h2048_i768_e128_k8", 2048, 768, 128, 8, (1, 2, 4, 8)),
    LayerShape("dsv3_h7168_i2048_e256_k8", 7168, 2048, 256, 8, (1, 2, 8, 16, 32)),
    LayerShape("dsv3_wide_h7168_i2048_e256_k8", 7168, 2048, 256, 8, (256, 512)),
    LayerShape("skewed_h4096_i1536_e128_k8", 4096, 1536, 128, 8, (1024,), skew_bias=True),
)


def config_seed(config_index: int, M: int) -> int:
    return 1000 * config_index + M


# --------------------------------------------------------------------------- splitmix64 (numpy)

def _mix_np(z: np.ndarray) -> np.ndarray:
    z = z ^ (z >> np.uint64(30))
    z = z * np.uint64(_MIX1)
    z = z ^ (z >> np.uint64(27))
    z = z * np.uint64(_MIX2)
    return z ^ (z >> np.uint64(31))


def _mix_int(z: int) -> int:
    z &= _MASK64
    z = ((z ^ (z >> 30)) * _MIX1) & _MASK64
    z = ((z ^ (z >> 27)) * _MIX2) & _MASK64
    return z ^ (z >> 31)


def stream_base(seed: int, tag: int, sub: int = 0) -> int:
    """64-bit base of the counter stream named by (seed, tag, sub)."""
    return _mix_int(_mix_int(_mix_int(seed * GAMMA + 1) ^ tag) + sub * GAMMA)


def _draws_np(base: int, start: int, count: int) -> np.ndarray:
    with np.errstate(over="ignore"):
        idx = np.arange(start + 1, start + 1 + count, dtype=np.uint64)
        return _mix_np(np.uint64(base) + idx * np.uint64(GAMMA))


# --------------------------------------------------------------------------- splitmix64 (torch)

def _to_i64(v: int) -> int:
    v &= _MASK64
    return v - (1 << 64) if v >= (1 << 63) else v


def _lsr_t(z, s: int):
    return (z >> s) & ((1 << (64 - s)) - 1)


def _mix_t(z):
    z = z ^ _lsr_t(z, 30)
    z = z * _to_i64(_MIX1)
    z = z ^ _lsr_t(z, 27)
    z = z * _to_i64(_MIX2)
    return z ^ _lsr_t(z, 31)


def _draws_t(base: int, start: int, count: int, device):
    import torch
    idx = torch.arange(start + 1, start + 1 + count, dtype=torch.int64, device=device)
    return _mix_t(idx * _to_i64(GAMMA) + _to_i64(base))


# --------------------------------------------------------------------------- integer streams

_CHUNK = 1 << 24   # draws per torch chunk (bounds device temporaries to ~0.5 GB)


def stream_bytes(base: int, byte_start: int, nbytes: int, backend: str = "numpy", device=None, out=None):
    """Bytes [byte_start, byte_start+nbytes) of a stream; byte b is bits 8*(b%8).. of draw b//8."""
    d0 = byte_start // 8
    d1 = (byte_start + nbytes + 7) // 8
    off = byte_start - 8 * d0
    if backend == "numpy":
        z = _draws_np(base, d0, d1 - d0)
        return z.view(np.uint8)[off:off + nbytes].copy()
    import torch
    if out is None:
        out = torch.empty(nbytes, dtype=torch.uint8, device=device)
    pos = 0
    d = d0
    while d < d1:
        n = min(_CHUNK, d1 - d)
        b = _draws_t(base, d, n, device).view(torch.uint8)
        lo = off if d == d0 else 0
        take = min(b.numel() - lo, nbytes - pos)
        out[pos:pos + take] = b[lo:lo + take]
        pos += take
        d += n
    return out


def stream_scale_codes(base: int, start: int, count: int, backend: str = "numpy", device=None, out=None):
    """E8M0 scale bytes uniform over {120..124}: 120 + floor(5 * hi32(draw) / 2^32)."""
    if backend == "numpy":
        z = _draws_np(base, start, count)
        return (np.uint64(SCALE_LO) + (((z >> np.uint64(32)) * np.uint64(SCALE_N)) >> np.uint64(32))).astype(np.uint8)
    import torch
    if out is None:
        out = torch.empty(count, dtype=torch.uint8, device=device)
    pos = 0
    while pos < count:
        n = min(_CHUNK, count - pos)
        z = _draws_t(base, start + pos, n, device)
        out[pos:pos + n] = (SCALE_LO + ((_lsr_t(z, 32) * SCALE_N) >> 32)).to(torch.uint8)
        pos += n
    return out


# --------------------------------------------------------------------------- floating streams (host only)

def _normals_np(base: int, count: int) -> np.ndarray:
    z = _draws_np(base, 0, 2 * count)
    u1 = ((z[0::2] >> np.uint64(11)).astype(np.float64) + 1.0) * 2.0 ** -53   # (0, 1]
    u2 = (z[1::2] >> np.uint64(11)).astype(np.float64) * 2.0 ** -53           # [0, 1)
    return np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * math.pi * u2)


def _bf16_bits_rne(v: np.ndarray) -> np.ndarray:
    """Round fp64 values (normal range) to bf16, round-to-nearest-even, return the 16-bit patterns."""
    m, e = np.frexp(v)                              # v = m * 2^e, 0.5 <= |m| < 1
    r = np.ldexp(np.round(m * 256.0), e - 8)        # 8 significant bits, ties to even
    return (r.astype(np.float32).view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def make_x(seed: int, M: int, H: int, attempts: Optional[Sequence[int]] = None) -> np.ndarray:
    """Token activations as bf16 bit patterns [M, H]; token t uses sub-stream (t, attempt[t])."""
    x = np.empty((M, H), dtype=np.uint16)
    for t in range(M):
        a = 0 if attempts is None else attempts[t]
        x[t] = _bf16_bits_rne(_normals_np(stream_base(seed, _TAG_X, (t << 16) | a), H))
    return x


def make_router(seed: int, H: int, E: int, skew_bias: bool):
    w = (_normals_np(stream_base(seed, _TAG_WR), E * H) / math.sqrt(H)).astype(np.float32).reshape(E, H)
    bias = None
    if skew_bias:
        # Zipf-like per-expert load: b_e = 3 * ln(1 / (e + 1))
        bias = np.array([3.0 * math.log(1.0 / (e + 1)) for e in range(E)], dtype=np.float32)
    return w, bias


def margin_ok(x_bits: np.ndarray, router_w: np.ndarray, bias, k: int) -> np.ndarray:
    """Per token: True when the k+1 largest fp64 logits are pairwise >= MARGIN apart."""
    logits = bf16_bits_to_f64(x_bits) @ router_w.astype(np.float64).T
    if bias is not None:
        logits = logits + bias.astype(np.float64)
    E = logits.shape[1]
    top = -np.sort(-logits, axis=1)[:, :min(k + 1, E)]
    gaps = top[:, :-1] - top[:, 1:]
    return np.all(gaps >= MARGIN, axis=1)


# --------------------------------------------------------------------------- weights

def expert_bytes(seed: int, which: str, e: int, rows: int, K: int, backend="numpy", device=None, out=None):
    """Packed E2M1 bytes of expert e: [rows, K/2] (w13: rows=2I, K=H; w2: rows=H, K=I)."""
    tag = _TAG_W13Q if which == "w13" else _TAG_W2Q
    n = rows * K // 2
    b = stream_bytes(stream_base(seed, tag), e * n, n, backend, device, out)
    return b.reshape(rows, K // 2) if out is None else out


def expert_scales(seed: int, which: str, e: int, rows: int, K: int, backend="numpy", device=None, out=None):
    """E8M0 scale bytes of expert e: [rows, K/32]."""
    tag = _TAG_W13S if which == "w13" else _TAG_W2S
    n = rows * K // 32
    s = stream_scale_codes(stream_base(seed, tag), e * n, n, backend, device, out)
    return s.reshape(rows, K // 32) if out is None else out


@dataclasses.dataclass
class MoEInputs:
    shape: LayerShape
    M: int
    seed: int
    x: np.ndarray                 # uint16 bf16 bits [M, H]
    router_w: np.ndarray          # float32 [E, H]
    router_bias: Optional[np.ndarray]
    attempts: list                # redraw attempt used per token
    w13_q: object = None          # [E, 2I, H/2] uint8 (numpy or torch)
    w13_s: object = None          # [E, 2I, H/32]
    w2_q: object = None           # [E, H, I/2]
    w2_s: object = None           # [E, H, I/32]

    def expert_weights(self, e: int):
        """One expert's (w13_q, w13_s, w2_q, w2_s) as host numpy arrays, regenerated from the streams."""
        s = self.shape
        return (expert_bytes(self.seed, "w13", e, 2 * s.I, s.H),
                expert_scales(self.seed, "w13", e, 2 * s.I, s.H),
                expert_bytes(self.seed, "w2", e, s.H, s.I),
                expert_scales(self.seed, "w2", e, s.H, s.I))


def make_inputs(config_index: int, M: Optional[int] = None, *, shape: Optional[LayerShape] = None,
                seed: Optional[int] = None, weights: str = "numpy", device=None) -> MoEInputs:
    """Build one workload.  weights: 'numpy' (host arrays), 'torch' (generated on `device`), or 'none'."""
    shape = shape or CONFIGS[config_index]
    M = shape.default_M if M is None else M
    seed = config_seed(config_index, M) if seed is None else seed
    H, I, E, k = shape.H, shape.I, shape.E, shape.k
    router_w, bias = make_router(seed, H, E, shape.skew_bias)
    attempts = [0] * M
    x = make_x(seed, M, H, attempts) if M > 0 else np.zeros((0, H), np.uint16)
    if M > 0:
        ok = margin_ok(x, router_w, bias, k)
        while not ok.all():
            for t in np.nonzero(~ok)[0]:
                attempts[t] += 1
                if attempts[t] > 1000:
                    raise RuntimeError("could not meet the routing margin")
                x[t] = _bf16_bits_rne(_normals_np(stream_base(seed, _TAG_X, (int(t) << 16) | attempts[t]), H))
            ok = margin_ok(x, router_w, bias, k)
    inp = MoEInputs(shape, M, seed, x, router_w, bias, attempts)
    if weights == "none":
        return inp
    if weights == "numpy":
        inp.w13_q = np.stack([expert_bytes(seed, "w13", e, 2 * I, H) for e in range(E)])
        inp.w13_s = np.stack([expert_scales(seed, "w13", e, 2 * I, H) for e in range(E)])
        inp.w2_q = np.stack([expert_bytes(seed, "w2", e, H, I) for e in range(E)])
        inp.w2_s = np.stack([expert_scales(seed, "w2", e, H, I) for e in range(E)])
        return inp
    import torch
    inp.w13_q = stream_bytes(stream_base(seed, _TAG_W13Q), 0, E * 2 * I * H // 2, "torch", device).view(E, 2 * I, H // 2)
    inp.w13_s = stream_scale_codes(stream_base(seed, _TAG_W13S), 0, E * 2 * I * H // 32, "torch", device).view(E, 2 * I, H // 32)
    inp.w2_q = stream_bytes(stream_base(seed, _TAG_W2Q), 0, E * H * I // 2, "torch", device).view(E, H, I // 2)
    inp.w2_s = stream_scale_codes(stream_base(seed, _TAG_W2S), 0, E * H * I // 32, "torch", device).view(E, H, I // 32)
    return inp
