"""Routed Mixture-of-Experts layer (Gemma-4-26B-A4B shapes, Q4_0 experts) on B200.

The compute lives in libmoe.so (hand-written sm_100a kernels behind a C ABI, declared in
include/moe.h). This package only marshals arguments to it; see `_lib`.
"""
from ._lib import (  # noqa: F401
    MOE_OK, MOE_ERR_NOT_INIT, MOE_ERR_BAD_ARG, MOE_ERR_BAD_ALIGN, MOE_ERR_CUDA,
    MOE_ERR_DEVICE_TIMEOUT, MOE_ERR_UNSUPPORTED_DEVICE, MOE_PATH_AUTO, MOE_PATH_GEMV,
    MOE_PATH_GEMM, MOE_PATH_GEMV_SPLIT, MoeError, lib, moe_init, moe_layer_forward, moe_rmsnorm_bf16,
    moe_stack_forward, moe_set_path, moe_destroy, moe_last_error, moe_debug_get_routing,
    moe_debug_get_hidden, moe_debug_check, moe_workspace_bytes, moe_profile_begin,
    moe_profile_end, PROF_GROUPS, EXPORTED, moe_layer_forward_static, moe_profile_kernel_launches,
    moe_layer_forward_static_check, moe_debug_set_wait_ns, moe_debug_inject, MOE_INJECT_NONE,
    MOE_INJECT_SKIP_ROUTER_ARRIVAL, moe_block_forward, moe_route, moe_experts_forward, moe_gather_rows,
    moe_combine_slots,
)
