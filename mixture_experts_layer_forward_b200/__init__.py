"""B200-native (sm_100a) forward pass of one mixture-of-experts layer.

The layer (Comet: Fine-grained Computation-communication Overlapping for Mixture-of-Experts,
§2.1 "MoE Structure") runs entirely in the CUDA kernels of ``libmoe_b200.so``; this package
only marshals arguments to its C ABI (include/moe.h). PyTorch supplies device memory and
streams. There is no CPU fallback: if the library is missing every call raises.

Public names mirror the C ABI: ``moe_workspace_size``, ``moe_padded_rows_max``,
``moe_route``, ``moe_dispatch``, ``moe_forward``, ``moe_forward_staged``,
``moe_forward_host``, ``moe_combine``, ``moe_get_device_status``.
"""
from ._native import (  # noqa: F401
    ACT_GELU_TANH,
    ACT_IDENTITY,
    ACT_RELU,
    ACT_SWIGLU,
    GATE_SOFTMAX_ALL,
    GATE_SELECT_BIAS,
    GATE_SOFTMAX_TOPK,
    MOE_NUM_STAGE_EVENTS,
    MoeError,
    Problem,
    library,
    library_path,
    moe_combine,
    moe_dispatch,
    moe_forward,
    moe_forward_host,
    moe_forward_host_batches,
    moe_forward_launches,
    moe_forward_staged,
    moe_get_device_status,
    moe_padded_rows_max,
    moe_route,
    moe_route_noalloc,
    moe_set_gemm_mode,
    moe_set_router_mode,
    moe_set_work_order,
    ORDER_EXPERT,
    ORDER_MIXED,
    ORDER_NARROW,
    ROUTER_AUTO,
    ROUTER_SEQUENTIAL,
    ROUTER_FILTER,
    moe_set_wait_timeout_ns,
    GEMM_AUTO,
    GEMM_FUSED,
    moe_set_fault_injection,
    GEMM_CTA_PAIR,
    GEMM_SINGLE_CTA,
    moe_workspace_size,
)
