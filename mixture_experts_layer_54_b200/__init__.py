"""Token-choice Mixture-of-Experts forward pass for NVIDIA B200 (sm_100a).

The work happens in libmoe_b200.so (CUDA kernels behind the C ABI of
include/moe_b200.h); this package is its ctypes binding.  Importing the ops
raises ImportError when the library has not been built.
"""
from ._abi import (MOE_ROW_ALIGN, CapacityFactorError, MoEError, MoeConfig, MoeOutputs,
                   MoeWeights, LIB_PATH, lib)
from .ops import (CapacityOut, HostStream, MoEForward, moe_bias_update, moe_capacity, moe_capacity_scored,
                  moe_seq_balance_loss, moe_clear_device_status, moe_probe_wait_timeout,
                  moe_dispatch_rows, moe_expert_ffn_gather, moe_expert_ffn_slots,
                  moe_combine_slots, moe_capacity_sharded,
                  gather_shard_counts, shard_losses, moe_capacity_noalloc, moe_capacity_value, moe_combine, moe_config,
                  moe_device_status, moe_dispatch, moe_expert_ffn, moe_forward,
                  moe_loss_partials_count, moe_losses, moe_perm_rows, moe_route,
                  moe_stage_workspace_size, moe_validate, moe_workspace_size, weights_struct,
                  StagedForward,
                  workspace)

__all__ = ["MOE_ROW_ALIGN", "CapacityFactorError", "MoEError", "MoeConfig", "MoeOutputs",
           "MoeWeights", "LIB_PATH", "lib", "CapacityOut", "HostStream", "MoEForward", "moe_bias_update",
           "moe_capacity_scored", "moe_seq_balance_loss", "moe_clear_device_status",
           "moe_probe_wait_timeout", "moe_dispatch_rows", "moe_expert_ffn_gather",
           "moe_expert_ffn_slots", "moe_combine_slots",
           "moe_capacity_sharded", "gather_shard_counts", "shard_losses", "moe_capacity", "moe_capacity_noalloc", "moe_capacity_value",
           "moe_combine", "moe_config", "moe_device_status", "moe_dispatch", "moe_expert_ffn",
           "moe_forward", "moe_loss_partials_count", "moe_losses", "moe_perm_rows", "moe_route",
           "moe_stage_workspace_size", "moe_validate", "moe_workspace_size", "weights_struct",
           "workspace", "StagedForward"]
