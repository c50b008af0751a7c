"""B200-native MoE expert-parallel token shuffle: route -> dispatch -> grouped SwiGLU FFN -> combine,
and its backward.

The stages are hand-written sm_100a CUDA kernels in ``libmoe.so`` behind the C ABI of
``include/moe.h``; this package is the thin Python binding (same names as the C entry points) plus
``MoeShuffle``, which owns the device buffers (allocated with torch) for one layer shape and calls
the entry points in order on one stream (forward, backward, CUDA-graph capture), and ``MoeEP``,
one expert-parallel layer over a process group.
"""
from ._lib import (EXPORTS, LIB_PATH, MOE_EP_PULL, MOE_EP_PUSH, MOE_ERR_CUDA, MOE_ERR_INVALID_ARG,
                   MOE_ERR_INVALID_COUNTS, MOE_ERR_INVALID_TOPK, MOE_ERR_TIMEOUT,
                   MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE, MOE_OK, MOE_PAYLOAD_BF16,
                   MOE_PAYLOAD_FP8_E4M3_B128, MoeError, load, moe_abi_version, moe_backward,
                   moe_backward_workspace_size, moe_capacity, moe_combine, moe_combine_backward,
                   moe_dispatch, moe_dispatch_noalloc, moe_dispatch_workspace_size, moe_ep_exchange,
                   moe_ep_regroup, moe_expert_backward, moe_expert_backward_workspace_size,
                   moe_expert_ffn, moe_expert_ffn_list, moe_expert_ffn_w8,
                   moe_ffn_w8_workspace_size, moe_ffn_weight_list_bytes, moe_ffn_weight_list_init,
                   moe_ffn_workspace_size, moe_quantize_rows_fp8, moe_route, moe_sync_status,
                   status_string)
from .layer import MoeShuffle
from .ep import MoeEP, TorchComm

__all__ = ["MoeShuffle", "MoeEP", "TorchComm", "MoeError", "load", "status_string", "EXPORTS",
           "LIB_PATH",
           # the C entry points
           "moe_abi_version", "moe_capacity", "moe_route", "moe_dispatch_workspace_size",
           "moe_dispatch", "moe_dispatch_noalloc", "moe_ffn_workspace_size", "moe_expert_ffn",
           "moe_ffn_weight_list_bytes", "moe_ffn_weight_list_init", "moe_expert_ffn_list",
           "moe_quantize_rows_fp8", "moe_ffn_w8_workspace_size", "moe_expert_ffn_w8",
           "moe_backward_workspace_size", "moe_backward", "moe_combine_backward",
           "moe_expert_backward_workspace_size", "moe_expert_backward", "moe_ep_regroup",
           "moe_ep_exchange", "moe_combine", "moe_sync_status",
           # status codes and constants
           "MOE_OK", "MOE_ERR_INVALID_ARG", "MOE_ERR_INVALID_TOPK", "MOE_ERR_UNSUPPORTED",
           "MOE_ERR_CUDA", "MOE_ERR_WORKSPACE", "MOE_ERR_TIMEOUT", "MOE_ERR_INVALID_COUNTS",
           "MOE_EP_PULL", "MOE_EP_PUSH", "MOE_PAYLOAD_BF16", "MOE_PAYLOAD_FP8_E4M3_B128"]
