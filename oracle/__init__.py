"""fp64 CPU oracle of the routed MXFP4 MoE layer -- TEST INFRASTRUCTURE ONLY.

Only `tests/`, `__graft_entry__.smoke()` and the CPU-baseline leg of `bench.py`
may import this package.  It wraps `moe_oracle.c` (plain C, fp64) through ctypes
and shares nothing with the CUDA library.  Parity of its full-layer output with
the pages is unpinned: the pages print no worked values for this layer; the
pins are closed forms, invariants and brute force (see tests/test_oracle_pins.py).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
# MOE_ORACLE_LIB: load another build of the same interface instead (the pins' mutation test loads
# copies of the oracle with one planted mistake each this way)
_LIB_OVERRIDE = os.environ.get("MOE_ORACLE_LIB")
_lib = None


def compile_lib(src: str, out: str) -> str:
    """gcc -O2 -fopenmp of one oracle source into a shared library (IEEE fp64, no fast-math)."""
    tmp = out + ".tmp%d" % os.getpid()
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-Wall", "-shared", "-fPIC", src, "-o", tmp, "-lm"])
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Compile moe_oracle.c into liboracle.so (gcc, -O2, OpenMP, IEEE fp64)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        compile_lib(_SRC, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        if _LIB_OVERRIDE:
            lib = ctypes.CDLL(_LIB_OVERRIDE)
        else:
            build()
            lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i = ctypes.c_int
        lib.oracle_e2m1_value.restype = ctypes.c_double
        lib.oracle_e2m1_value.argtypes = [i]
        lib.oracle_e8m0_scale.restype = ctypes.c_double
        lib.oracle_e8m0_scale.argtypes = [i]
        lib.oracle_mxfp4_weight.restype = ctypes.c_double
        lib.oracle_mxfp4_weight.argtypes = [P, P, i, ctypes.c_long, i]
        lib.oracle_bf16_to_double.restype = ctypes.c_double
        lib.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
        lib.oracle_round_bf16.restype = ctypes.c_uint16
        lib.oracle_round_bf16.argtypes = [ctypes.c_double]
        lib.oracle_route.restype = None
        lib.oracle_route.argtypes = [P, P, P, i, i, i, i, P, P, P]
        lib.oracle_permute.restype = None
        lib.oracle_permute.argtypes = [P, i, i, i, P, P, P]
        lib.oracle_expert_swiglu.restype = None
        lib.oracle_expert_swiglu.argtypes = [P, P, P, i, i, P, P, P]
        lib.oracle_expert_down.restype = None
        lib.oracle_expert_down.argtypes = [P, P, P, i, i, P]
        lib.oracle_forward.restype = None
        lib.oracle_forward.argtypes = [P, P, P, P, P, P, P, i, i, i, i, i, P, i, P, P, P, P, P]
        lib.oracle_num_threads.restype = i
        lib.oracle_set_num_threads.argtypes = [i]
        _lib = lib
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


# --------------------------------------------------------------------------- scalar formats

def e2m1_value(code: int) -> float:
    return _load().oracle_e2m1_value(int(code))


def e8m0_scale(byte: int) -> float:
    return _load().oracle_e8m0_scale(int(byte))


def mxfp4_weight(q: np.ndarray, s: np.ndarray, row: int, k: int) -> float:
    q = _c(q, np.uint8)
    s = _c(s, np.uint8)
    return _load().oracle_mxfp4_weight(_p(q), _p(s), q.shape[-1] * 2, row, k)


def round_bf16(v: float) -> int:
    return int(_load().oracle_round_bf16(float(v)))


def bf16_to_double(bits: int) -> float:
    return _load().oracle_bf16_to_double(int(bits))


def num_threads() -> int:
    return _load().oracle_num_threads()


def set_num_threads(n: int) -> None:
    _load().oracle_set_num_threads(int(n))


# --------------------------------------------------------------------------- layer steps

def route(x_bits: np.ndarray, router_w: np.ndarray, router_bias, k: int):
    """Router select/normalize: returns (topk_ids [M,k] int32, topk_w [M,k] f64, logits [M,E] f64)."""
    x = _c(x_bits, np.uint16)
    w = _c(router_w, np.float32)
    b = _c(router_bias, np.float32)
    M, H = x.shape
    E = w.shape[0]
    ids = np.zeros((M, k), np.int32)
    tw = np.zeros((M, k), np.float64)
    logits = np.zeros((M, E), np.float64)
    _load().oracle_route(_p(x), _p(w), _p(b), M, H, E, k, _p(ids), _p(tw), _p(logits))
    return ids, tw, logits


def permute(topk_ids: np.ndarray, E: int):
    """Route remap: returns (expert_offsets [E+1], sorted_ids [M*k], inv_pos [M*k]), int32."""
    ids = _c(topk_ids, np.int32)
    M, k = ids.shape
    off = np.zeros(E + 1, np.int32)
    srt = np.zeros(M * k, np.int32)
    inv = np.zeros(M * k, np.int32)
    _load().oracle_permute(_p(ids), M, E, k, _p(off), _p(srt), _p(inv))
    return off, srt, inv


def expert_swiglu(x_row, w13_q_e, w13_s_e):
    """One token through one expert's gate_up + clamp-SwiGLU: (g f64 [I], u f64 [I], h bf16 bits [I])."""
    x = _c(x_row, np.uint16)
    q = _c(w13_q_e, np.uint8)
    s = _c(w13_s_e, np.uint8)
    H = x.shape[-1]
    I = q.shape[0] // 2
    g = np.zeros(I, np.float64)
    u = np.zeros(I, np.float64)
    h = np.zeros(I, np.uint16)
    _load().oracle_expert_swiglu(_p(x), _p(q), _p(s), H, I, _p(g), _p(u), _p(h))
    return g, u, h


def expert_down(h_row, w2_q_e, w2_s_e):
    """One bf16 intermediate row through one expert's down projection: y f64 [H]."""
    h = _c(h_row, np.uint16)
    q = _c(w2_q_e, np.uint8)
    s = _c(w2_s_e, np.uint8)
    H = q.shape[0]
    I = h.shape[-1]
    y = np.zeros(H, np.float64)
    _load().oracle_expert_down(_p(h), _p(q), _p(s), H, I, _p(y))
    return y


def forward(x_bits, router_w, router_bias, w13_q, w13_s, w2_q, w2_s, k: int, tokens=None, I=None):
    """Full layer.  The four weight arguments are either [E, ...] arrays or dicts {expert: array}
    holding at least every expert the listed tokens route to.  Returns a dict with
    topk_ids, topk_w, h (bf16 bits, flat order t*k+j), out64, out_bf16 (bits)."""
    x = _c(x_bits, np.uint16)
    w = _c(router_w, np.float32)
    b = _c(router_bias, np.float32)
    M, H = x.shape
    E = w.shape[0]

    def table(src):
        keep = []
        arr = (ctypes.c_void_p * E)()
        for e in range(E):
            a = src.get(e) if isinstance(src, dict) else src[e]
            if a is None:
                continue
            a = _c(a, np.uint8)
            keep.append(a)
            arr[e] = a.ctypes.data
        return arr, keep

    t13q, k1 = table(w13_q)
    t13s, k2 = table(w13_s)
    t2q, k3 = table(w2_q)
    t2s, k4 = table(w2_s)
    if I is None:
        I = (w13_q[next(iter(w13_q))] if isinstance(w13_q, dict) else w13_q[0]).shape[0] // 2
    tok = None if tokens is None else np.ascontiguousarray(tokens, dtype=np.int32)
    ntok = 0 if tok is None else tok.size
    ids = np.zeros((M, k), np.int32)
    tw = np.zeros((M, k), np.float64)
    h = np.zeros((M * k, I), np.uint16)
    out64 = np.zeros((M, H), np.float64)
    outb = np.zeros((M, H), np.uint16)
    _load().oracle_forward(_p(x), _p(w), _p(b), t13q, t13s, t2q, t2s, M, H, I, E, k,
                           _p(tok), ntok, _p(ids), _p(tw), _p(h), _p(out64), _p(outb))
    del k1, k2, k3, k4
    return {"topk_ids": ids, "topk_w": tw, "h": h, "out64": out64, "out_bf16": outb}
