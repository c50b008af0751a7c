"""Device buffers for one MoE layer shape and the four C-ABI calls in order on one stream.

Memory comes from torch (the caller-owned allocation of the C ABI); all arithmetic runs in
libmoe.so.  Nothing here synchronises with the host except ``status()``.
"""
from __future__ import annotations

import torch

from . import _lib


def expect(t, shape, dtype, name: str, device=None) -> None:
    """Raise unless ``t`` is a contiguous tensor of this shape and dtype (on ``device`` if given).

    The kernels trust these shapes (a short ``x`` would be read past its end), so every tensor a
    caller hands to ``MoeShuffle`` is checked here, on the host, before anything is launched.
    """
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor, got {type(t).__name__}")
    if t.dtype != dtype:
        raise TypeError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous (row-major)")
    if device is not None and t.device != device:
        raise ValueError(f"{name}: on {t.device}, expected {device}")


class MoeShuffle:
    """Route -> dispatch -> grouped SwiGLU FFN -> combine for T tokens of width H over E experts.

    ``payload`` is "bf16" or "fp8" (e4m3 codes + one fp32 scale per 128 elements); ``capacity``
    is the per-expert row limit (0 = keep every slot, see ``moe_capacity``); rank r of R owns
    experts [r*E/R, (r+1)*E/R).
    """

    def __init__(self, T: int, H: int, E: int, k: int, R: int, F: int, payload: str = "bf16",
                 capacity: int = 0, renormalize: bool = True, device="cuda"):
        _lib.load()
        self.T, self.H, self.E, self.k, self.R, self.F = T, H, E, k, R, F
        self.capacity = int(capacity)
        self.renormalize = bool(renormalize)
        self.fp8 = payload == "fp8"
        if payload not in ("bf16", "fp8"):
            raise ValueError("payload must be 'bf16' or 'fp8'")
        self.payload = _lib.MOE_PAYLOAD_FP8_E4M3_B128 if self.fp8 else _lib.MOE_PAYLOAD_BF16
        dev = torch.device(device)
        if dev.type == "cuda" and dev.index is None:
            dev = torch.device("cuda", torch.cuda.current_device())
        self.device = dev
        i32 = dict(dtype=torch.int32, device=dev)
        S = T * k
        self.max_rows = S
        self.topk_idx = torch.empty((T, k), **i32)
        self.topk_w = torch.empty((T, k), dtype=torch.float32, device=dev)
        self.expert_routed = torch.empty(E, **i32)
        if self.fp8:
            self.send = torch.empty((S, H), dtype=torch.uint8, device=dev)
            self.send_scales = torch.empty((S, H // 128), dtype=torch.float32, device=dev)
        else:
            self.send = torch.empty((S, H), dtype=torch.bfloat16, device=dev)
            self.send_scales = None
        self.expert_counts = torch.empty(E, **i32)
        self.expert_offsets = torch.empty(E + 1, **i32)
        self.rank_offsets = torch.empty(R + 1, **i32)
        self.slot_row = torch.empty((T, k), **i32)
        self.row_token = torch.empty(max(S, 1), **i32)
        self.expert_out = torch.empty((S, H), dtype=torch.bfloat16, device=dev)
        self.y = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
        self.ws_dispatch_bytes = _lib.moe_dispatch_workspace_size(T, E, k)
        self.ws_dispatch = torch.zeros(self.ws_dispatch_bytes, dtype=torch.uint8, device=dev)
        self.ws_ffn_bytes = _lib.moe_ffn_workspace_size(S, E, H, F, self.payload)
        self.ws_ffn = torch.zeros(self.ws_ffn_bytes, dtype=torch.uint8, device=dev)
        self.ws_ffn_w8 = None  # allocated by the first expert_ffn_w8 call

    # -- views into the FFN workspace ----------------------------------------------------------
    @property
    def h(self) -> torch.Tensor:
        """The bf16 SwiGLU intermediate [max_rows, F] (inside the FFN workspace)."""
        n = self.max_rows * self.F * 2
        return self.ws_ffn[256:256 + n].view(torch.bfloat16).view(self.max_rows, self.F)

    # -- the four stages ----------------------------------------------------------------------
    def route(self, logits: torch.Tensor, stream=None):
        expect(logits, (self.T, self.E), torch.float32, "logits", self.device)
        _lib.moe_route(logits, self.T, self.E, self.k, self.renormalize, self.topk_idx,
                       self.topk_w, self.expert_routed, stream)

    def dispatch(self, x: torch.Tensor, topk_idx: torch.Tensor | None = None, stream=None):
        idx = self.topk_idx if topk_idx is None else topk_idx
        expect(x, (self.T, self.H), torch.bfloat16, "x", self.device)
        expect(idx, (self.T, self.k), torch.int32, "topk_idx", self.device)
        _lib.moe_dispatch(x, self.T, self.H, idx, self.k, self.E, self.R, self.capacity,
                          self.payload, self.send, self.send_scales, self.expert_counts,
                          self.expert_offsets, self.rank_offsets, self.slot_row, self.row_token,
                          self.ws_dispatch, self.ws_dispatch_bytes, stream)

    def expert_ffn(self, w_gate, w_up, w_down, send=None, send_scales=None, expert_offsets=None,
                   stream=None):
        bf16 = torch.bfloat16
        expect(w_gate, (self.E, self.F, self.H), bf16, "w_gate", self.device)
        expect(w_up, (self.E, self.F, self.H), bf16, "w_up", self.device)
        expect(w_down, (self.E, self.H, self.F), bf16, "w_down", self.device)
        if send is not None:
            expect(send, (self.max_rows, self.H), self.send.dtype, "send", self.device)
        if send_scales is not None:
            expect(send_scales, (self.max_rows, self.H // 128), torch.float32, "send_scales",
                   self.device)
        if expert_offsets is not None:
            expect(expert_offsets, (self.E + 1,), torch.int32, "expert_offsets", self.device)
        _lib.moe_expert_ffn(self.send if send is None else send,
                            self.send_scales if send_scales is None else send_scales,
                            self.payload,
                            self.expert_offsets if expert_offsets is None else expert_offsets,
                            self.max_rows, self.E, self.H, self.F, w_gate, w_up, w_down,
                            self.expert_out, self.ws_ffn, self.ws_ffn_bytes, stream)

    def expert_weight_list(self, w_gate, w_up, w_down) -> torch.Tensor:
        """Device descriptors of per-expert weights at separate addresses (sequences of E tensors
        [F,H], [F,H], [H,F] bf16); the weights must stay where they are while the list is used."""
        for e in range(self.E):
            expect(w_gate[e], (self.F, self.H), torch.bfloat16, f"w_gate[{e}]", self.device)
            expect(w_up[e], (self.F, self.H), torch.bfloat16, f"w_up[{e}]", self.device)
            expect(w_down[e], (self.H, self.F), torch.bfloat16, f"w_down[{e}]", self.device)
        n = _lib.moe_ffn_weight_list_bytes(self.E)
        wlist = torch.empty(n, dtype=torch.uint8, device=self.device)
        _lib.moe_ffn_weight_list_init(list(w_gate), list(w_up), list(w_down), self.E, self.H,
                                      self.F, wlist)
        torch.cuda.synchronize(self.device)
        return wlist

    def expert_ffn_list(self, wlist, send=None, send_scales=None, expert_offsets=None, stream=None):
        """expert_ffn with the weights of ``expert_weight_list``."""
        expect(wlist, (_lib.moe_ffn_weight_list_bytes(self.E),), torch.uint8, "wlist", self.device)
        if send is not None:
            expect(send, (self.max_rows, self.H), self.send.dtype, "send", self.device)
        if send_scales is not None:
            expect(send_scales, (self.max_rows, self.H // 128), torch.float32, "send_scales",
                   self.device)
        if expert_offsets is not None:
            expect(expert_offsets, (self.E + 1,), torch.int32, "expert_offsets", self.device)
        _lib.moe_expert_ffn_list(self.send if send is None else send,
                                 self.send_scales if send_scales is None else send_scales,
                                 self.payload,
                                 self.expert_offsets if expert_offsets is None else expert_offsets,
                                 self.max_rows, self.E, self.H, self.F, wlist, self.expert_out,
                                 self.ws_ffn, self.ws_ffn_bytes, stream)

    def quantize_expert_weights_fp8(self, w_gate, w_up):
        """FP8 gate / up weights for ``expert_ffn_w8``: (gate codes, gate scales, up codes, up
        scales), e4m3 [E,F,H] with one fp32 scale per row [E,F].  Set-up, outside the step."""
        expect(w_gate, (self.E, self.F, self.H), torch.bfloat16, "w_gate", self.device)
        expect(w_up, (self.E, self.F, self.H), torch.bfloat16, "w_up", self.device)
        out = []
        for w in (w_gate, w_up):
            q = torch.empty((self.E, self.F, self.H), dtype=torch.uint8, device=self.device)
            sc = torch.empty((self.E, self.F), dtype=torch.float32, device=self.device)
            _lib.moe_quantize_rows_fp8(w, self.E * self.F, self.H, q, sc)
            out += [q, sc]
        return tuple(out)

    def expert_ffn_w8(self, w_gate_q, w_gate_scale, w_up_q, w_up_scale, w_down, send=None,
                      send_scales=None, expert_offsets=None, stream=None):
        """expert_ffn with FP8 gate / up weights (``quantize_expert_weights_fp8``) and bf16 down
        weights; the FFN input rows are quantised to FP8 per row inside the call."""
        expect(w_gate_q, (self.E, self.F, self.H), torch.uint8, "w_gate_q", self.device)
        expect(w_up_q, (self.E, self.F, self.H), torch.uint8, "w_up_q", self.device)
        expect(w_gate_scale, (self.E, self.F), torch.float32, "w_gate_scale", self.device)
        expect(w_up_scale, (self.E, self.F), torch.float32, "w_up_scale", self.device)
        expect(w_down, (self.E, self.H, self.F), torch.bfloat16, "w_down", self.device)
        if send is not None:
            expect(send, (self.max_rows, self.H), self.send.dtype, "send", self.device)
        if send_scales is not None:
            expect(send_scales, (self.max_rows, self.H // 128), torch.float32, "send_scales",
                   self.device)
        if expert_offsets is not None:
            expect(expert_offsets, (self.E + 1,), torch.int32, "expert_offsets", self.device)
        if self.ws_ffn_w8 is None:
            n = _lib.moe_ffn_w8_workspace_size(self.max_rows, self.E, self.H, self.F, self.payload)
            self.ws_ffn_w8 = torch.zeros(n, dtype=torch.uint8, device=self.device)
        _lib.moe_expert_ffn_w8(self.send if send is None else send,
                               self.send_scales if send_scales is None else send_scales,
                               self.payload,
                               self.expert_offsets if expert_offsets is None else expert_offsets,
                               self.max_rows, self.E, self.H, self.F, w_gate_q, w_gate_scale,
                               w_up_q, w_up_scale, w_down, self.expert_out, self.ws_ffn_w8,
                               self.ws_ffn_w8.numel(), stream)

    @property
    def h_w8(self) -> torch.Tensor:
        """The bf16 SwiGLU intermediate of the last ``expert_ffn_w8`` call [max_rows, F]."""
        n = self.max_rows * self.F * 2
        return self.ws_ffn_w8[256:256 + n].view(torch.bfloat16).view(self.max_rows, self.F)

    def combine(self, expert_out=None, slot_row=None, topk_w=None, stream=None):
        if expert_out is not None:
            expect(expert_out, (self.max_rows, self.H), torch.bfloat16, "expert_out", self.device)
        if slot_row is not None:
            expect(slot_row, (self.T, self.k), torch.int32, "slot_row", self.device)
        if topk_w is not None:
            expect(topk_w, (self.T, self.k), torch.float32, "topk_w", self.device)
        # the combine has no device-side waits and no device-side findings: no status word
        _lib.moe_combine(self.expert_out if expert_out is None else expert_out, self.max_rows,
                         self.slot_row if slot_row is None else slot_row,
                         self.topk_w if topk_w is None else topk_w, self.T, self.k, self.H,
                         self.y, None, stream)

    # -- backward ------------------------------------------------------------------------------
    def backward(self, dy, logits, w_gate, w_up, w_down, stream=None) -> dict:
        """Gradients for the output gradient ``dy`` [T,H] bf16, after ``forward`` on the same
        tensors (its routing, plan, FFN input rows and expert outputs are reused).  Returns a dict
        of dx bf16 [T,H], d_logits fp32 [T,E], d_topk_w fp32 [T,k], d_w_gate / d_w_up fp32
        [E,F,H], d_w_down fp32 [E,H,F] (buffers owned by this object, overwritten by the next
        call)."""
        bf16, f32 = torch.bfloat16, torch.float32
        expect(dy, (self.T, self.H), bf16, "dy", self.device)
        expect(logits, (self.T, self.E), f32, "logits", self.device)
        expect(w_gate, (self.E, self.F, self.H), bf16, "w_gate", self.device)
        expect(w_up, (self.E, self.F, self.H), bf16, "w_up", self.device)
        expect(w_down, (self.E, self.H, self.F), bf16, "w_down", self.device)
        if getattr(self, "grads", None) is None:
            dev = self.device
            self.grads = {
                "dx": torch.empty((self.T, self.H), dtype=bf16, device=dev),
                "d_logits": torch.empty((self.T, self.E), dtype=f32, device=dev),
                "d_topk_w": torch.empty((self.T, self.k), dtype=f32, device=dev),
                "d_w_gate": torch.empty((self.E, self.F, self.H), dtype=f32, device=dev),
                "d_w_up": torch.empty((self.E, self.F, self.H), dtype=f32, device=dev),
                "d_w_down": torch.empty((self.E, self.H, self.F), dtype=f32, device=dev),
            }
            n = _lib.moe_backward_workspace_size(self.max_rows, self.T, self.k, self.H, self.F)
            self.ws_bwd = torch.zeros(n, dtype=torch.uint8, device=dev)
        g = self.grads
        ffn_input = self.send if not self.fp8 else self.dequantized_rows
        _lib.moe_backward(dy, self.T, self.H, self.k, self.E, self.F, logits, self.renormalize,
                          self.topk_idx, self.topk_w, self.slot_row, self.expert_offsets,
                          self.max_rows, ffn_input, self.expert_out, w_gate, w_up, w_down,
                          g["dx"], g["d_logits"], g["d_topk_w"], g["d_w_gate"], g["d_w_up"],
                          g["d_w_down"], self.ws_bwd, self.ws_bwd.numel(), stream)
        return g

    def backward_intermediate(self, name: str) -> torch.Tensor:
        """A view into the backward workspace: "d_eo", "dx_rows" [max_rows, H] or "h", "dg",
        "du" [max_rows, F] (bf16), as the last ``backward`` left them."""
        up = lambda b: (b + 255) // 256 * 256  # noqa: E731
        r, H, F = max(self.max_rows, 1), self.H, self.F
        sizes = [("d_eo", r * H * 2, H), ("h", r * F * 2, F), ("dg", r * F * 2, F),
                 ("du", r * F * 2, F), ("dx_rows", r * H * 2, H)]
        off = 256
        for key, nbytes, cols in sizes:
            if key == name:
                return self.ws_bwd[off:off + nbytes].view(torch.bfloat16).view(r, cols)
            off += up(nbytes)
        raise KeyError(name)

    @property
    def dequantized_rows(self) -> torch.Tensor:
        """The FP8 payload's bf16 FFN input rows [max_rows, H] (in the FFN workspace, after h)."""
        up = lambda b: (b + 255) // 256 * 256  # noqa: E731
        off = 256 + up(self.max_rows * self.F * 2)
        n = self.max_rows * self.H * 2
        return self.ws_ffn[off:off + n].view(torch.bfloat16).view(self.max_rows, self.H)

    def forward(self, logits, x, w_gate, w_up, w_down, stream=None) -> torch.Tensor:
        self.route(logits, stream)
        self.dispatch(x, stream=stream)
        self.expert_ffn(w_gate, w_up, w_down, stream=stream)
        self.combine(stream=stream)
        return self.y

    def capture(self, logits, x, w_gate, w_up, w_down, out=None) -> torch.cuda.CUDAGraph:
        """Record ``forward`` on these exact tensors (and, if given, ``out.copy_(y)``) as a CUDA graph.

        ``replay()`` of the returned graph reruns the whole step with one launch from the host: new
        inputs are written into the same ``logits`` / ``x`` tensors before each replay.  The step
        allocates nothing and never synchronises, and the FFN's counters return to zero inside
        every call, so a replay needs no reset.  One eager call runs first, outside the capture.
        """
        self.forward(logits, x, w_gate, w_up, w_down)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        # thread-local capture: other threads of the process (a communicator's watchdog, say) may
        # keep making CUDA calls while this thread records
        with torch.cuda.graph(g, capture_error_mode="thread_local"):
            self.forward(logits, x, w_gate, w_up, w_down)
            if out is not None:
                out.copy_(self.y)
        return g

    def capture_step(self, logits, x, w_gate, w_up, w_down, dy) -> torch.cuda.CUDAGraph:
        """Record a training step, ``forward`` then ``backward`` for the output gradient ``dy``, on
        these exact tensors as one CUDA graph (neither half synchronises with the host).  Each
        ``replay()`` reruns both with whatever ``logits`` / ``x`` / ``dy`` (and the weights) hold;
        the gradients land in ``self.grads``.  One eager step runs first, outside the capture."""
        self.forward(logits, x, w_gate, w_up, w_down)
        self.backward(dy, logits, w_gate, w_up, w_down)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, capture_error_mode="thread_local"):
            self.forward(logits, x, w_gate, w_up, w_down)
            self.backward(dy, logits, w_gate, w_up, w_down)
        return g

    def status(self, stream=None) -> int:
        """Synchronise and return (then clear) the device status of the dispatch, FFN and backward
        stages."""
        found = [_lib.moe_sync_status(self.ws_dispatch, stream),
                 _lib.moe_sync_status(self.ws_ffn, stream)]
        if self.ws_ffn_w8 is not None:
            found.append(_lib.moe_sync_status(self.ws_ffn_w8, stream))
        if getattr(self, "ws_bwd", None) is not None:
            found.append(_lib.moe_sync_status(self.ws_bwd, stream))
        return next((st for st in found if st != _lib.MOE_OK), _lib.MOE_OK)
