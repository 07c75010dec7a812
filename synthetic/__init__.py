"""Seeded synthetic inputs for the MoE layer (activations, router, quantised experts).

This package is input generation only. It draws random tensors and encodes
expert weights into the stored formats (E2M1/E8M0, E2M1/E4M3, E4M3, bf16).
It holds none of the layer's forward arithmetic (no decode, routing, FFN or
combine): both the CUDA path and the CPU oracle consume what it produces.
"""
from .gen import (  # noqa: F401
    CONFIGS,
    LayerInputs,
    WFMT,
    make_layer,
    make_router,
    make_tokens,
    zipf_bias,
    expert_bytes,
    quantise,
)
