"""B200-native routed Mixture-of-Experts decode block (Flash-MoE hot path) and Gated DeltaNet
state update for sm_100a.

The compute lives in libfmoe.so (hand-written CUDA kernels behind the C ABI of
include/fmoe.h, fmoe_gdn.h and fmoe_cache.h); this package is its thin Python binding.
"""
from ._abi import (FmoeBank, FmoeError, FmoeExpertCache, FmoeLayer, Bank, ExpertCache, Layer, GDN_STATE_EARLY,
                   bank_layout, expert_ffn, expert_ffn_workspace_size, gdn_step, lib, moe_layer, moe_layer_cached,
                   moe_layer_routed, moe_layer_static, moe_layer_workspace_size, moe_stack, rmsnorm, router_topk,
                   router_topk_workspace_size, trace_next_layer, wait_flag, workspace, workspace_check, workspace_init)

__all__ = ["FmoeBank", "FmoeError", "FmoeExpertCache", "FmoeLayer", "Bank", "ExpertCache", "Layer", "GDN_STATE_EARLY",
           "bank_layout", "expert_ffn", "expert_ffn_workspace_size", "gdn_step", "lib", "moe_layer", "moe_layer_cached",
           "moe_layer_routed", "moe_layer_static",
           "moe_layer_workspace_size", "moe_stack", "rmsnorm", "router_topk", "router_topk_workspace_size",
           "trace_next_layer", "wait_flag", "workspace", "workspace_check", "workspace_init"]
