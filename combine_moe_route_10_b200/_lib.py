"""ctypes binding of libmoe.so (include/moe.h).  Argument marshalling only: every step of the path
runs in the library's CUDA kernels; there is no CPU fallback and loading fails loudly when the
library is missing."""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoe.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_INVALID_TOPK = 2
MOE_ERR_UNSUPPORTED = 3
MOE_ERR_CUDA = 4
MOE_ERR_WORKSPACE = 5
MOE_ERR_TIMEOUT = 6
MOE_ERR_INVALID_COUNTS = 7
MOE_EP_PULL = 0
MOE_EP_PUSH = 1
MOE_PAYLOAD_BF16 = 0
MOE_PAYLOAD_FP8_E4M3_B128 = 1

EXPORTS = ["moe_abi_version", "moe_status_string", "moe_capacity", "moe_route",
           "moe_dispatch_workspace_size", "moe_dispatch", "moe_dispatch_noalloc",
           "moe_ffn_workspace_size",
           "moe_expert_ffn", "moe_ffn_weight_list_bytes", "moe_ffn_weight_list_init",
           "moe_expert_ffn_list", "moe_quantize_rows_fp8", "moe_ffn_w8_workspace_size",
           "moe_expert_ffn_w8", "moe_backward_workspace_size", "moe_backward", "moe_combine_backward", "moe_expert_backward_workspace_size", "moe_expert_backward", "moe_ep_regroup", "moe_ep_exchange", "moe_combine", "moe_sync_status"]

_lib = None


class MoeError(RuntimeError):
    def __init__(self, status: int, call: str):
        self.status = status
        super().__init__(f"{call}: {status_string(status)}")


def load() -> ctypes.CDLL:
    """Load libmoe.so (built by ``python -m combine_moe_route_10_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libmoe.so not found at {LIB_PATH}; build it with "
                          "`python -m combine_moe_route_10_b200.build` (nvcc, sm_100a)")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, Z, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_double
    sig = {
        "moe_abi_version": (I, []),
        "moe_status_string": (ctypes.c_char_p, [I]),
        "moe_capacity": (I, [D, I, I, I]),
        "moe_route": (I, [P, I, I, I, I, P, P, P, P]),
        "moe_dispatch_workspace_size": (Z, [I, I, I]),
        "moe_dispatch": (I, [P, I, I, P, I, I, I, I, I, P, P, P, P, P, P, P, P, Z, P]),
        "moe_dispatch_noalloc": (I, [P, I, I, P, I, I, I, I, I, P, P, P, P, P, P, P, P, P]),
        "moe_ffn_workspace_size": (Z, [I, I, I, I, I]),
        "moe_expert_ffn": (I, [P, P, I, P, I, I, I, I, P, P, P, P, P, Z, P]),
        "moe_ffn_weight_list_bytes": (Z, [I]),
        "moe_ffn_weight_list_init": (I, [P, P, P, I, I, I, P, P]),
        "moe_expert_ffn_list": (I, [P, P, I, P, I, I, I, I, P, P, P, Z, P]),
        "moe_quantize_rows_fp8": (I, [P, I, I, P, P, P]),
        "moe_ffn_w8_workspace_size": (Z, [I, I, I, I, I]),
        "moe_expert_ffn_w8": (I, [P, P, I, P, I, I, I, I, P, P, P, P, P, P, P, Z, P]),
        "moe_backward_workspace_size": (Z, [I, I, I, I, I]),
        "moe_backward": (I, [P, I, I, I, I, I, P, I, P, P, P, P, I, P, P, P, P, P, P, P, P, P, P,
                             P, P, Z, P]),
        "moe_combine_backward": (I, [P, I, I, I, I, P, I, P, P, P, I, P, P, P, P, P]),
        "moe_expert_backward_workspace_size": (Z, [I, I]),
        "moe_expert_backward": (I, [P, P, P, I, I, I, I, P, P, P, P, P, P, P, P, Z, P]),
        "moe_ep_regroup": (I, [P, I, I, I, I, I, I, I, I, P, P, Z, P, P, Z, P, P, P]),
        "moe_ep_exchange": (I, [P, I, I, I, I, P, P, I, P, P, I, Z, Z, P, P, P]),
        "moe_combine": (I, [P, I, P, P, I, I, I, P, P, P]),
        "moe_sync_status": (I, [P, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load().moe_status_string(int(status)).decode()


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(st: int, call: str, raise_on_error: bool):
    if raise_on_error and st != MOE_OK:
        raise MoeError(st, call)
    return st


def moe_abi_version() -> int:
    return load().moe_abi_version()


def moe_capacity(cf: float, T: int, k: int, E: int) -> int:
    return load().moe_capacity(float(cf), T, k, E)


def moe_route(logits, T, E, k, renormalize, topk_idx, topk_w, expert_routed=None, stream=None,
              raise_on_error=True):
    st = load().moe_route(_ptr(logits), T, E, k, int(renormalize), _ptr(topk_idx), _ptr(topk_w),
                          _ptr(expert_routed), _stream(stream))
    return _check(st, "moe_route", raise_on_error)


def moe_dispatch_workspace_size(T, E, k) -> int:
    return load().moe_dispatch_workspace_size(T, E, k)


def moe_dispatch(x, T, H, topk_idx, k, E, R, capacity, payload, send, send_scales, expert_counts,
                 expert_offsets, rank_offsets, slot_row, row_token, ws, ws_bytes, stream=None,
                 raise_on_error=True):
    st = load().moe_dispatch(_ptr(x), T, H, _ptr(topk_idx), k, E, R, capacity, payload, _ptr(send),
                             _ptr(send_scales), _ptr(expert_counts), _ptr(expert_offsets),
                             _ptr(rank_offsets), _ptr(slot_row), _ptr(row_token), _ptr(ws),
                             ws_bytes, _stream(stream))
    return _check(st, "moe_dispatch", raise_on_error)


def moe_dispatch_noalloc(x, T, H, topk_idx, k, E, R, capacity, payload, send, send_scales,
                         expert_counts, expert_offsets, rank_offsets, slot_row, row_token,
                         status=None, stream=None, raise_on_error=True):
    """moe_dispatch without a workspace: for callers that cannot allocate device memory (the
    library keeps a 1 MiB static device array for the scratch; see include/moe.h)."""
    st = load().moe_dispatch_noalloc(_ptr(x), T, H, _ptr(topk_idx), k, E, R, capacity, payload,
                                     _ptr(send), _ptr(send_scales), _ptr(expert_counts),
                                     _ptr(expert_offsets), _ptr(rank_offsets), _ptr(slot_row),
                                     _ptr(row_token), _ptr(status), _stream(stream))
    return _check(st, "moe_dispatch_noalloc", raise_on_error)


def moe_ffn_workspace_size(max_rows, E, H, F, payload) -> int:
    return load().moe_ffn_workspace_size(max_rows, E, H, F, payload)


def moe_expert_ffn(send, send_scales, payload, expert_offsets, max_rows, E, H, F, w_gate, w_up,
                   w_down, expert_out, ws, ws_bytes, stream=None, raise_on_error=True):
    st = load().moe_expert_ffn(_ptr(send), _ptr(send_scales), payload, _ptr(expert_offsets),
                               max_rows, E, H, F, _ptr(w_gate), _ptr(w_up), _ptr(w_down),
                               _ptr(expert_out), _ptr(ws), ws_bytes, _stream(stream))
    return _check(st, "moe_expert_ffn", raise_on_error)


def moe_ffn_weight_list_bytes(E) -> int:
    return load().moe_ffn_weight_list_bytes(E)


def moe_ffn_weight_list_init(w_gate, w_up, w_down, E, H, F, wlist, stream=None,
                             raise_on_error=True):
    """Per-expert weight descriptors into the device buffer ``wlist``: w_gate / w_up / w_down are
    sequences of E per-expert tensors ([F,H], [F,H], [H,F] bf16, each its own allocation)."""
    arr = ctypes.c_void_p * E
    g = arr(*[_ptr(t) for t in w_gate])
    u = arr(*[_ptr(t) for t in w_up])
    d = arr(*[_ptr(t) for t in w_down])
    st = load().moe_ffn_weight_list_init(ctypes.cast(g, ctypes.c_void_p),
                                         ctypes.cast(u, ctypes.c_void_p),
                                         ctypes.cast(d, ctypes.c_void_p), E, H, F, _ptr(wlist),
                                         _stream(stream))
    return _check(st, "moe_ffn_weight_list_init", raise_on_error)


def moe_expert_ffn_list(send, send_scales, payload, expert_offsets, max_rows, E, H, F, wlist,
                        expert_out, ws, ws_bytes, stream=None, raise_on_error=True):
    st = load().moe_expert_ffn_list(_ptr(send), _ptr(send_scales), payload, _ptr(expert_offsets),
                                    max_rows, E, H, F, _ptr(wlist), _ptr(expert_out), _ptr(ws),
                                    ws_bytes, _stream(stream))
    return _check(st, "moe_expert_ffn_list", raise_on_error)


def moe_quantize_rows_fp8(x, rows, K, codes, scales, stream=None, raise_on_error=True):
    st = load().moe_quantize_rows_fp8(_ptr(x), rows, K, _ptr(codes), _ptr(scales), _stream(stream))
    return _check(st, "moe_quantize_rows_fp8", raise_on_error)


def moe_ffn_w8_workspace_size(max_rows, E, H, F, payload) -> int:
    return load().moe_ffn_w8_workspace_size(max_rows, E, H, F, payload)


def moe_expert_ffn_w8(send, send_scales, payload, expert_offsets, max_rows, E, H, F, w_gate_q,
                      w_gate_scale, w_up_q, w_up_scale, w_down, expert_out, ws, ws_bytes,
                      stream=None, raise_on_error=True):
    st = load().moe_expert_ffn_w8(_ptr(send), _ptr(send_scales), payload, _ptr(expert_offsets),
                                  max_rows, E, H, F, _ptr(w_gate_q), _ptr(w_gate_scale),
                                  _ptr(w_up_q), _ptr(w_up_scale), _ptr(w_down), _ptr(expert_out),
                                  _ptr(ws), ws_bytes, _stream(stream))
    return _check(st, "moe_expert_ffn_w8", raise_on_error)


def moe_backward_workspace_size(max_rows, T, k, H, F) -> int:
    return load().moe_backward_workspace_size(max_rows, T, k, H, F)


def moe_backward(dy, T, H, k, E, F, logits, renormalize, topk_idx, topk_w, slot_row,
                 expert_offsets, max_rows, ffn_input, expert_out, w_gate, w_up, w_down, dx,
                 d_logits, d_topk_w, d_w_gate, d_w_up, d_w_down, ws, ws_bytes, stream=None,
                 raise_on_error=True):
    st = load().moe_backward(_ptr(dy), T, H, k, E, F, _ptr(logits), int(renormalize),
                             _ptr(topk_idx), _ptr(topk_w), _ptr(slot_row), _ptr(expert_offsets),
                             max_rows, _ptr(ffn_input), _ptr(expert_out), _ptr(w_gate),
                             _ptr(w_up), _ptr(w_down), _ptr(dx), _ptr(d_logits), _ptr(d_topk_w),
                             _ptr(d_w_gate), _ptr(d_w_up), _ptr(d_w_down), _ptr(ws), ws_bytes,
                             _stream(stream))
    return _check(st, "moe_backward", raise_on_error)


def moe_combine_backward(dy, T, H, k, E, logits, renormalize, topk_idx, topk_w, slot_row,
                         max_rows, expert_out, d_eo, d_topk_w, d_logits, stream=None,
                         raise_on_error=True):
    st = load().moe_combine_backward(_ptr(dy), T, H, k, E, _ptr(logits), int(renormalize),
                                     _ptr(topk_idx), _ptr(topk_w), _ptr(slot_row), max_rows,
                                     _ptr(expert_out), _ptr(d_eo), _ptr(d_topk_w), _ptr(d_logits),
                                     _stream(stream))
    return _check(st, "moe_combine_backward", raise_on_error)


def moe_expert_backward_workspace_size(max_rows, F) -> int:
    return load().moe_expert_backward_workspace_size(max_rows, F)


def moe_expert_backward(ffn_input, d_eo, expert_offsets, max_rows, E, H, F, w_gate, w_up, w_down,
                        dx_rows, d_w_gate, d_w_up, d_w_down, ws, ws_bytes, stream=None,
                        raise_on_error=True):
    st = load().moe_expert_backward(_ptr(ffn_input), _ptr(d_eo), _ptr(expert_offsets), max_rows, E,
                                    H, F, _ptr(w_gate), _ptr(w_up), _ptr(w_down), _ptr(dx_rows),
                                    _ptr(d_w_gate), _ptr(d_w_up), _ptr(d_w_down), _ptr(ws),
                                    ws_bytes, _stream(stream))
    return _check(st, "moe_expert_backward", raise_on_error)


def moe_ep_regroup(counts, A, B, src_order, src_stride, src_rows, dst_order, dst_stride, dst_rows,
                   src, dst, row_bytes, src_aux=None, dst_aux=None, aux_row_bytes=0,
                   dst_offsets=None, status=None, stream=None, raise_on_error=True):
    st = load().moe_ep_regroup(_ptr(counts), A, B, src_order, src_stride, src_rows, dst_order,
                               dst_stride, dst_rows, _ptr(src), _ptr(dst), row_bytes,
                               _ptr(src_aux), _ptr(dst_aux), aux_row_bytes, _ptr(dst_offsets),
                               _ptr(status), _stream(stream))
    return _check(st, "moe_ep_regroup", raise_on_error)


def moe_ep_exchange(all_counts, R, E, rank, direction, peer_rows, peer_aux, peer_rows_cap,
                    local_rows, local_aux, local_rows_cap, row_bytes, aux_row_bytes=0,
                    local_offsets=None, status=None, stream=None, raise_on_error=True):
    st = load().moe_ep_exchange(_ptr(all_counts), R, E, rank, direction, _ptr(peer_rows),
                                _ptr(peer_aux), peer_rows_cap, _ptr(local_rows), _ptr(local_aux),
                                local_rows_cap, row_bytes, aux_row_bytes, _ptr(local_offsets),
                                _ptr(status), _stream(stream))
    return _check(st, "moe_ep_exchange", raise_on_error)


def moe_combine(expert_out, max_rows, slot_row, topk_w, T, k, H, y, status=None, stream=None,
                raise_on_error=True):
    st = load().moe_combine(_ptr(expert_out), max_rows, _ptr(slot_row), _ptr(topk_w), T, k, H,
                            _ptr(y), _ptr(status), _stream(stream))
    return _check(st, "moe_combine", raise_on_error)


def moe_sync_status(ws, stream=None) -> int:
    return load().moe_sync_status(_ptr(ws), _stream(stream))
