"""B200-native (sm_100a) fused Mixture-of-Experts layer.

route top-k -> atomic-free permutation -> tcgen05 grouped SwiGLU GEMMs
(expert-weight rows in the MMA M slot, tokens in N) -> weighted combine,
behind the C ABI of include/moe.h, and the CPU/GPU expert split of
include/moe_split.h.  This package is the thin ctypes binding.
"""
from ._lib import (HOST_ISA_AMX_BF16, HOST_ISA_AVX512_BF16, HOST_ISA_PORTABLE, POLICY_ALL_CPU, POLICY_ALL_STAGED,
                   POLICY_BALANCED, POLICY_DYNAMIC, SPLIT_CPU, SPLIT_IDLE, SPLIT_RESIDENT, SPLIT_STAGED,
                   SplitCosts, SplitLayer, host_expert_ffn, host_isa, host_pack_weights,
                   host_packed_size, split_costs, split_place, split_plan)
from ._lib import (BF16, COMBINE_AUTO, COMBINE_DETERMINISTIC, COMBINE_FUSED, FP8_E4M3, Lora, MoEError, MoELayer, align_permute, check_status, combine,
                   forward, forward_workspace_size, grouped_ffn, grouped_ffn_workspace_size, lib,
                   pack_weights, permute_capacity, route_topk, selftest_wait_timeout,
                   status_string, version, LIB_PATH)

__all__ = ["BF16", "COMBINE_AUTO", "COMBINE_DETERMINISTIC", "COMBINE_FUSED", "FP8_E4M3", "Lora", "MoEError", "MoELayer", "align_permute", "check_status", "combine",
           "forward", "forward_workspace_size", "grouped_ffn", "grouped_ffn_workspace_size", "lib",
           "pack_weights", "permute_capacity", "route_topk", "selftest_wait_timeout",
           "status_string", "version", "LIB_PATH",
           "HOST_ISA_AMX_BF16", "HOST_ISA_AVX512_BF16", "HOST_ISA_PORTABLE", "POLICY_ALL_CPU", "POLICY_ALL_STAGED",
           "POLICY_BALANCED", "POLICY_DYNAMIC", "SPLIT_CPU", "SPLIT_IDLE", "SPLIT_RESIDENT", "SPLIT_STAGED",
           "SplitCosts", "SplitLayer", "host_expert_ffn", "host_isa", "host_pack_weights",
           "host_packed_size", "split_costs", "split_place", "split_plan"]
