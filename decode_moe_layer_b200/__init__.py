"""B200-native routed MXFP4 Mixture-of-Experts layer for LLM decode.

The compute lives in libmoe.so (hand-written CUDA for sm_100a, C ABI in
include/moe.h); this package is its thin Python binding.  Importing it loads
the library and fails loudly if it has not been built.
"""
from ._lib import (  # noqa: F401
    EXPORTS,
    LIB_PATH,
    MOE_ERR_CUDA,
    MOE_ERR_INVALID_ARG,
    MOE_ERR_TIMEOUT,
    MOE_ERR_UNSUPPORTED_SHAPE,
    MOE_ERR_WORKSPACE,
    MOE_OK,
    MoEError,
    load,
    moe_down_combine,
    moe_forward_launches,
    moe_gate_up_swiglu,
    moe_mxfp4_forward,
    moe_mxfp4_forward_ex,
    moe_mxfp4_forward_partial,
    moe_mxfp4_forward_profile,
    PROFILE_KERNELS,
    moe_permute,
    moe_reduce_partials,
    moe_route,
    moe_route_noalloc,
    moe_selftest_wait_timeout,
    moe_status_string,
    moe_workspace_bytes,
)

load()
