"""Routed-expert MoE layer (softmax top-k, batch union, int4 gs64 x Q8_0 SwiGLU
experts, shared expert, weighted combine) for NVIDIA B200 (sm_100a).

The compute lives in libmoe.so (C ABI, include/moe.h); this package is its thin
ctypes binding.  Build the library with
``python -m int4_routed_expert_softmax_b200.build``.
"""
from ._lib import (  # noqa: F401
    MOE_DECODE_T_MAX, MOE_OK, MOE_PATH_AUTO, MOE_PATH_DECODE, MOE_PATH_PREFILL, MoeDims, MoeError,
    alloc_workspace, dims, expert_table, lib, moe_bucket, moe_check_dims, moe_device_binary_version,
    moe_device_sms, moe_layer_launches, moe_set_wait_limit,
    moe_expert_bytes, moe_layer_forward, moe_layer_forward_static, moe_layer_forward_mxfp4, moe_profile_enable, moe_profile_read, moe_layer_forward_host, moe_quant_q8_0, moe_router_topk,
    moe_workspace_bytes, moe_workspace_bytes_path, moe_workspace_view, status_string, ws_slice,
)
