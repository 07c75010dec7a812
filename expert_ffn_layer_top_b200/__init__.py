"""B200 (sm_100a) MoE layer forward over quantised experts.

Thin Python binding of libmoe.so (include/moe.h): every function here only
marshals arguments (torch tensors -> device pointers, the current CUDA stream)
and allocates outputs with torch; all the arithmetic runs in the library's
CUDA kernels. There is no fallback: if the library cannot be loaded, every call
raises.
"""
from ._lib import (  # noqa: F401
    ACT,
    FMT,
    ExpertCache,
    Experts,
    MoeError,
    lib,
    moe_combine,
    moe_dequantize,
    moe_device_error,
    moe_grouped_ffn,
    moe_layer_forward,
    moe_permute,
    moe_permute_static,
    moe_prepack,
    moe_selftest_wait,
    moe_tensor_peak_tflops,
    moe_set_wait_limit_ns,
    PREFETCH,
    moe_prepacked_expert_bytes,
    LAYOUT_STANDARD,
    LAYOUT_TILED,
    moe_route_topk,
    moe_version,
    moe_kernel_launch_count,
    moe_workspace_size,
)
