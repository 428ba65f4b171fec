"""B200-native routed Mixture-of-Experts decode block (Flash-MoE hot path) for sm_100a.

The compute lives in libfmoe.so (hand-written CUDA kernels behind the C ABI of
include/fmoe.h); this package is its thin Python binding.
"""
from ._abi import (FmoeBank, FmoeError, FmoeLayer, Bank, Layer, bank_layout, expert_ffn, expert_ffn_workspace_size,
                   lib, moe_layer, moe_layer_routed, moe_layer_static, moe_layer_workspace_size, moe_stack, rmsnorm,
                   router_topk, router_topk_workspace_size, trace_next_layer, wait_flag, workspace, workspace_check,
                   workspace_init)

__all__ = ["FmoeBank", "FmoeError", "FmoeLayer", "Bank", "Layer", "bank_layout", "expert_ffn",
           "expert_ffn_workspace_size", "lib", "moe_layer", "moe_layer_routed", "moe_layer_static",
           "moe_layer_workspace_size", "moe_stack", "rmsnorm", "router_topk", "router_topk_workspace_size",
           "trace_next_layer", "wait_flag", "workspace", "workspace_check", "workspace_init"]
