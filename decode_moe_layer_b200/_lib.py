"""ctypes binding of libmoe.so.  Argument marshalling only: every step of the layer
runs in the library's CUDA kernels; this module allocates outputs with torch and
passes raw device pointers, sizes and the current CUDA stream."""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = -1
MOE_ERR_UNSUPPORTED_SHAPE = -2
MOE_ERR_WORKSPACE = -3
MOE_ERR_CUDA = -4
MOE_ERR_TIMEOUT = -5

# every symbol include/moe.h declares
EXPORTS = (
    "moe_status_string", "moe_last_cuda_error", "moe_route", "moe_permute", "moe_gate_up_swiglu",
    "moe_down_combine", "moe_mxfp4_forward", "moe_workspace_bytes", "moe_forward_launches", "moe_mxfp4_forward_ex",
    "moe_mxfp4_forward_profile", "moe_route_noalloc", "moe_selftest_wait_timeout", "moe_mxfp4_forward_partial",
    "moe_reduce_partials",
)
PROFILE_KERNELS = ("route_logits", "route_select", "permute", "gate_up", "gather", "gate_up_tc_small",
                   "gate_up_tc_large", "down", "down_tc_small", "down_tc_large", "combine")

_lib = None


class MoEError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        name = load().moe_status_string(status).decode()
        extra = ""
        if status == MOE_ERR_CUDA:
            extra = " (cudaError %d)" % load().moe_last_cuda_error()
        super().__init__("%s returned %s%s" % (where, name, extra))


def load():
    """Load libmoe.so; raises if it has not been built (there is no fallback path)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError("libmoe.so not built: run `python decode_moe_layer_b200/build.py` (needs nvcc)")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    lib.moe_status_string.restype = ctypes.c_char_p
    lib.moe_status_string.argtypes = [I]
    lib.moe_last_cuda_error.restype = I
    lib.moe_last_cuda_error.argtypes = []
    lib.moe_route.restype = I
    lib.moe_route.argtypes = [P, P, P, P, P, I, I, I, I, P]
    lib.moe_route_noalloc.restype = I
    lib.moe_route_noalloc.argtypes = [P, P, P, P, P, I, I, I, I, P]
    lib.moe_permute.restype = I
    lib.moe_permute.argtypes = [P, P, P, P, I, I, I, P]
    lib.moe_gate_up_swiglu.restype = I
    lib.moe_gate_up_swiglu.argtypes = [P, P, P, P, P, P, I, I, I, I, I, P]
    lib.moe_down_combine.restype = I
    lib.moe_down_combine.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, P]
    lib.moe_mxfp4_forward.restype = I
    lib.moe_mxfp4_forward.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, P]
    lib.moe_workspace_bytes.restype = S
    lib.moe_workspace_bytes.argtypes = [I, I, I, I, I]
    lib.moe_forward_launches.restype = I
    lib.moe_forward_launches.argtypes = [I, I, I, I, I]
    lib.moe_mxfp4_forward_ex.restype = I
    lib.moe_mxfp4_forward_ex.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, P, P, P, P, S, P]
    lib.moe_mxfp4_forward_profile.restype = I
    lib.moe_mxfp4_forward_profile.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, P, P, P, P, S, P, P]
    lib.moe_selftest_wait_timeout.restype = I
    lib.moe_selftest_wait_timeout.argtypes = [P, P]
    lib.moe_mxfp4_forward_partial.restype = I
    lib.moe_mxfp4_forward_partial.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, P, P, P, P, S, P]
    lib.moe_reduce_partials.restype = I
    lib.moe_reduce_partials.argtypes = [P, I, P, I, I, P]
    _lib = lib
    return lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(rc: int, where: str):
    if rc != MOE_OK:
        raise MoEError(rc, where)


def _need(t, dtype, name):
    if t.dtype != dtype or not t.is_cuda or not t.is_contiguous():
        raise ValueError("%s must be a contiguous CUDA %s tensor" % (name, dtype))


# --------------------------------------------------------------------------- API (same names as the C ABI)

def moe_status_string(status: int) -> str:
    return load().moe_status_string(int(status)).decode()


def moe_workspace_bytes(M: int, H: int, I: int, E: int, k: int) -> int:
    return int(load().moe_workspace_bytes(M, H, I, E, k))


def moe_forward_launches(M: int, H: int, I: int, E: int, k: int) -> int:
    """Kernel launches of one layer call for this shape (negative MOE_* status if unsupported)."""
    return int(load().moe_forward_launches(M, H, I, E, k))


def moe_selftest_wait_timeout(status_out, stream=None):
    """Launch the bounded-wait self-test: writes MOE_ERR_TIMEOUT into status_out (int32 [1], CUDA)."""
    _need(status_out, torch.int32, "status_out")
    _check(load().moe_selftest_wait_timeout(_ptr(status_out), _stream(stream)), "moe_selftest_wait_timeout")


def moe_route(x, router_w, k: int, router_bias=None, stream=None):
    """x bf16 [M,H], router_w fp32 [E,H] -> (topk_ids int32 [M,k], topk_w fp32 [M,k])."""
    _need(x, torch.bfloat16, "x")
    _need(router_w, torch.float32, "router_w")
    M, H = x.shape
    E = router_w.shape[0]
    ids = torch.empty((M, k), dtype=torch.int32, device=x.device)
    w = torch.empty((M, k), dtype=torch.float32, device=x.device)
    rc = load().moe_route(_ptr(x), _ptr(router_w), _ptr(router_bias), _ptr(ids), _ptr(w), M, H, E, k, _stream(stream))
    _check(rc, "moe_route")
    return ids, w


def moe_route_noalloc(x, router_w, k: int, router_bias=None, stream=None):
    """moe_route with its scratch in the library's static device array (no device allocation)."""
    _need(x, torch.bfloat16, "x")
    _need(router_w, torch.float32, "router_w")
    M, H = x.shape
    E = router_w.shape[0]
    ids = torch.empty((M, k), dtype=torch.int32, device=x.device)
    w = torch.empty((M, k), dtype=torch.float32, device=x.device)
    rc = load().moe_route_noalloc(_ptr(x), _ptr(router_w), _ptr(router_bias), _ptr(ids), _ptr(w), M, H, E, k,
                                  _stream(stream))
    _check(rc, "moe_route_noalloc")
    return ids, w


def moe_permute(topk_ids, E: int, stream=None):
    """topk_ids int32 [M,k] -> (expert_offsets [E+1], sorted_ids [M*k], inv_pos [M*k]), int32."""
    _need(topk_ids, torch.int32, "topk_ids")
    M, k = topk_ids.shape
    dev = topk_ids.device
    off = torch.empty(E + 1, dtype=torch.int32, device=dev)
    srt = torch.empty(M * k, dtype=torch.int32, device=dev)
    inv = torch.empty(M * k, dtype=torch.int32, device=dev)
    rc = load().moe_permute(_ptr(topk_ids), _ptr(off), _ptr(srt), _ptr(inv), M, E, k, _stream(stream))
    _check(rc, "moe_permute")
    return off, srt, inv


def moe_gate_up_swiglu(x, w13_q, w13_s, expert_offsets, sorted_ids, k: int, stream=None):
    """-> h bf16 [M*k, I] in expert-grouped order (row p = assignment sorted_ids[p])."""
    _need(x, torch.bfloat16, "x")
    M, H = x.shape
    E, I2, _ = w13_q.shape
    I = I2 // 2
    h = torch.empty((M * k, I), dtype=torch.bfloat16, device=x.device)
    rc = load().moe_gate_up_swiglu(_ptr(x), _ptr(w13_q), _ptr(w13_s), _ptr(expert_offsets), _ptr(sorted_ids),
                                   _ptr(h), M, H, I, E, k, _stream(stream))
    _check(rc, "moe_gate_up_swiglu")
    return h


def moe_down_combine(h, w2_q, w2_s, topk_w, expert_offsets, sorted_ids, M: int, k: int, stream=None):
    """h bf16 [M*k, I] (expert-grouped, as moe_gate_up_swiglu writes it) -> out bf16 [M, H]."""
    _need(h, torch.bfloat16, "h")
    E, H, _ = w2_q.shape
    I = h.shape[1]
    out = torch.empty((M, H), dtype=torch.bfloat16, device=h.device)
    rc = load().moe_down_combine(_ptr(h), _ptr(w2_q), _ptr(w2_s), _ptr(topk_w), _ptr(expert_offsets),
                                 _ptr(sorted_ids), _ptr(out), M, H, I, E, k, _stream(stream))
    _check(rc, "moe_down_combine")
    return out


def moe_mxfp4_forward(x, router_w, w13_q, w13_s, w2_q, w2_s, k: int, out=None, stream=None):
    """Whole layer with the library-owned workspace: -> out bf16 [M, H]."""
    _need(x, torch.bfloat16, "x")
    M, H = x.shape
    E, I2, _ = w13_q.shape
    if out is None:
        out = torch.empty((M, H), dtype=torch.bfloat16, device=x.device)
    rc = load().moe_mxfp4_forward(_ptr(x), _ptr(router_w), _ptr(w13_q), _ptr(w13_s), _ptr(w2_q), _ptr(w2_s),
                                  _ptr(out), M, H, I2 // 2, E, k, _stream(stream))
    _check(rc, "moe_mxfp4_forward")
    return out


def moe_mxfp4_forward_ex(x, router_w, w13_q, w13_s, w2_q, w2_s, k: int, workspace, router_bias=None, out=None,
                         topk_ids_out=None, topk_w_out=None, status_out=None, stream=None):
    """Whole layer with a caller-owned workspace (uint8 CUDA tensor of >= moe_workspace_bytes)."""
    _need(x, torch.bfloat16, "x")
    M, H = x.shape
    E, I2, _ = w13_q.shape
    if out is None:
        out = torch.empty((M, H), dtype=torch.bfloat16, device=x.device)
    rc = load().moe_mxfp4_forward_ex(_ptr(x), _ptr(router_w), _ptr(router_bias), _ptr(w13_q), _ptr(w13_s),
                                     _ptr(w2_q), _ptr(w2_s), _ptr(out), M, H, I2 // 2, E, k, _ptr(topk_ids_out),
                                     _ptr(topk_w_out), _ptr(status_out), _ptr(workspace),
                                     0 if workspace is None else workspace.numel() * workspace.element_size(),
                                     _stream(stream))
    _check(rc, "moe_mxfp4_forward_ex")
    return out


def moe_mxfp4_forward_partial(x, router_w, w13_q, w13_s, w2_q, w2_s, k: int, workspace, router_bias=None,
                              partial_out=None, topk_ids_out=None, topk_w_out=None, status_out=None, stream=None):
    """One rank's fp32 share [M,H] of an I-sharded layer; the weights are the rank's slices
    (w13 [E, 2*I_shard, H/2], w2 [E, H, I_shard/2], as sharded.shard_weights returns them)."""
    _need(x, torch.bfloat16, "x")
    M, H = x.shape
    E, I2, _ = w13_q.shape
    if partial_out is None:
        partial_out = torch.empty((M, H), dtype=torch.float32, device=x.device)
    _need(partial_out, torch.float32, "partial_out")
    rc = load().moe_mxfp4_forward_partial(_ptr(x), _ptr(router_w), _ptr(router_bias), _ptr(w13_q), _ptr(w13_s),
                                          _ptr(w2_q), _ptr(w2_s), _ptr(partial_out), M, H, I2 // 2, E, k,
                                          _ptr(topk_ids_out), _ptr(topk_w_out), _ptr(status_out), _ptr(workspace),
                                          0 if workspace is None else workspace.numel() * workspace.element_size(),
                                          _stream(stream))
    _check(rc, "moe_mxfp4_forward_partial")
    return partial_out


def moe_reduce_partials(partials, out=None, stream=None):
    """out [M,H] bf16 = bf16(sum over g ascending of partials[g]) for partials [G,M,H] fp32."""
    _need(partials, torch.float32, "partials")
    G, M, H = partials.shape
    if out is None:
        out = torch.empty((M, H), dtype=torch.bfloat16, device=partials.device)
    _need(out, torch.bfloat16, "out")
    rc = load().moe_reduce_partials(_ptr(partials), G, _ptr(out), M, H, _stream(stream))
    _check(rc, "moe_reduce_partials")
    return out


def moe_mxfp4_forward_profile(x, router_w, w13_q, w13_s, w2_q, w2_s, k: int, workspace, router_bias=None,
                              out=None, stream=None):
    """Whole layer plus per-kernel device times: -> (out, {kernel name: ms}).  Synchronises the stream."""
    _need(x, torch.bfloat16, "x")
    M, H = x.shape
    E, I2, _ = w13_q.shape
    if out is None:
        out = torch.empty((M, H), dtype=torch.bfloat16, device=x.device)
    ms = (ctypes.c_float * len(PROFILE_KERNELS))()
    rc = load().moe_mxfp4_forward_profile(_ptr(x), _ptr(router_w), _ptr(router_bias), _ptr(w13_q), _ptr(w13_s),
                                          _ptr(w2_q), _ptr(w2_s), _ptr(out), M, H, I2 // 2, E, k, None, None, None,
                                          _ptr(workspace), workspace.numel() * workspace.element_size(),
                                          _stream(stream), ms)
    _check(rc, "moe_mxfp4_forward_profile")
    return out, {name: float(ms[i]) for i, name in enumerate(PROFILE_KERNELS)}
