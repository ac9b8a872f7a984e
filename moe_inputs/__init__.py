"""Seeded synthetic inputs for the routed MXFP4 MoE layer.

This module is shared by the CPU oracle (tests) and the CUDA path (tests, bench).
It holds none of the layer's arithmetic: it only draws inputs with the shapes,
value distributions and routing structure of the decode workloads.
"""
from .generator import (  # noqa: F401
    CONFIGS,
    LayerShape,
    MoEInputs,
    make_inputs,
    make_x,
    make_router,
    expert_bytes,
    expert_scales,
    stream_bytes,
    stream_scale_codes,
    margin_ok,
)
