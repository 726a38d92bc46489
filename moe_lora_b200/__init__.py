"""moe_lora_b200: batched multi-tenant LoRA on a Mixture-of-Experts FFN, for B200.

The computation lives in libmoe_lora.so (CUDA, sm_100a), behind the C ABI declared
in include/moe_lora.h; this package is its thin Python binding (torch tensors in,
torch tensors out, the current torch CUDA stream).
"""
from ._lib import (AdapterFormat, ERR_CUDA, ERR_DEVICE_CHECK, ERR_INVALID_ARG, ERR_TIMEOUT, ERR_UNSUPPORTED, EXPORTS,
                   LIB_PATH, ML_BF16, ML_E4M3, ML_F32, OK, OP_DENSE, OP_FORWARD, OP_FORWARD_BF16,
                   OP_FORWARD_E4M3, OP_ROUTE, OP_SGMV_EXPAND,
                   OP_SGMV_SHRINK, KERNEL_IDS, MoELoRAError, check_status, launch_count, profile_enable, profile_read, dense_lora_forward, forward, lib,
                   new_workspace, route, sgmv_expand, sgmv_shrink, version, workspace_size)

__all__ = ["AdapterFormat", "route", "forward", "sgmv_shrink", "sgmv_expand", "dense_lora_forward", "workspace_size",
           "new_workspace", "check_status", "version", "lib", "MoELoRAError", "EXPORTS", "LIB_PATH",
           "OK", "ERR_INVALID_ARG", "ERR_UNSUPPORTED", "ERR_CUDA", "ERR_DEVICE_CHECK", "ERR_TIMEOUT",
           "ML_F32", "ML_BF16", "ML_E4M3", "OP_ROUTE", "OP_FORWARD", "OP_FORWARD_BF16", "OP_FORWARD_E4M3",
           "OP_SGMV_SHRINK", "OP_SGMV_EXPAND",
           "OP_DENSE", "KERNEL_IDS", "profile_enable", "profile_read", "launch_count"]
