"""B200-native MoE expert-parallel token shuffle: route -> dispatch -> grouped SwiGLU FFN -> combine.

The four stages are hand-written sm_100a CUDA kernels in ``libmoe.so`` behind the C ABI of
``include/moe.h``; this package is the thin Python binding (same names as the C entry points) plus
``MoeShuffle``, which owns the device buffers (allocated with torch) for one layer shape and calls
the four entry points in order on one stream.
"""
from ._lib import (EXPORTS, LIB_PATH, MOE_ERR_CUDA, MOE_ERR_INVALID_ARG, MOE_ERR_INVALID_TOPK,
                   MOE_ERR_TIMEOUT, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE, MOE_OK,
                   MOE_PAYLOAD_BF16, MOE_PAYLOAD_FP8_E4M3_B128, MoeError, load, moe_abi_version,
                   moe_capacity, moe_combine, moe_dispatch, moe_dispatch_noalloc,
                   moe_dispatch_workspace_size,
                   moe_expert_ffn, moe_expert_ffn_list, moe_ffn_weight_list_bytes,
                   moe_ffn_weight_list_init, moe_ffn_workspace_size, moe_expert_ffn_w8,
                   moe_ffn_w8_workspace_size, moe_quantize_rows_fp8, moe_route, moe_sync_status,
                   status_string)
from .layer import MoeShuffle
from .ep import MoeEP, TorchComm
from ._lib import MOE_ERR_INVALID_COUNTS, moe_ep_regroup

__all__ = ["MoeShuffle", "MoeEP", "TorchComm", "moe_ep_regroup", "MOE_ERR_INVALID_COUNTS",
           "MoeError", "load", "moe_route", "moe_dispatch", "moe_expert_ffn",
           "moe_expert_ffn_list", "moe_ffn_weight_list_bytes", "moe_ffn_weight_list_init",
           "moe_expert_ffn_w8", "moe_ffn_w8_workspace_size", "moe_quantize_rows_fp8",
           "moe_combine", "moe_sync_status", "moe_dispatch_noalloc", "moe_capacity", "moe_dispatch_workspace_size",
           "moe_ffn_workspace_size", "moe_abi_version", "status_string", "EXPORTS", "LIB_PATH",
           "MOE_OK", "MOE_ERR_INVALID_ARG", "MOE_ERR_INVALID_TOPK", "MOE_ERR_UNSUPPORTED",
           "MOE_ERR_CUDA", "MOE_ERR_WORKSPACE", "MOE_ERR_TIMEOUT", "MOE_PAYLOAD_BF16",
           "MOE_PAYLOAD_FP8_E4M3_B128"]
