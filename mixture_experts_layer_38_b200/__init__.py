"""B200 (sm_100a) implementation of the LongCat-Flash MoE layer with zero-computation experts.

The work happens in libmoe_b200.so (C ABI: include/moe.h); this package is its thin binding
(:mod:`.binding`) plus the seeded synthetic workloads (:mod:`.workloads`).
"""
from .binding import (RENORMALIZE_GATES, Dims, MoeError, PidParams, alloc_workspace, dims,
                      moe_bias_update, moe_combine, moe_dense_ffn, moe_dispatch, moe_expert_ffn,
                      moe_expert_ffn_fp8, moe_expert_ffn_gather, moe_forward, moe_forward_fp8,
                      moe_last_device_error, moe_quantize_fp8, moe_route,
                      quantize_expert_weights_fp8, scratch_size, strerror, workspace_size)

__all__ = [
    "RENORMALIZE_GATES", "Dims", "MoeError", "PidParams", "alloc_workspace", "dims",
    "moe_bias_update", "moe_combine", "moe_dense_ffn", "moe_dispatch", "moe_expert_ffn", "moe_expert_ffn_fp8",
    "moe_expert_ffn_gather", "moe_forward", "moe_forward_fp8", "moe_last_device_error",
    "moe_quantize_fp8", "moe_route", "quantize_expert_weights_fp8", "scratch_size", "strerror",
    "workspace_size",
]
