"""Expert parallelism over a process group: one process per GPU, rank r owns experts
[r*E_loc, (r+1)*E_loc) with E_loc = E / R, and the rows cross the ranks in two all-to-alls.

One step on every rank, on its own T tokens (the NCCL EP page, sections 1 and 2: a dispatch
exchange to the experts' owners and a combine exchange back; the ThunderEP page, section 2.1:
one contiguous block per destination):

  1. route + dispatch with R ranks: the send buffer is destination-major, expert-major inside a
     destination's block; ``rank_offsets`` are the send displacements and ``expert_counts`` viewed
     as [R, E_loc] are the per-(destination, expert) row counts;
  2. all-to-all of those counts: rank r learns ``recv_counts[s][e]``, the rows source s sends to
     its local expert e;
  3. all-to-all of the rows (and, for the FP8 payload, their block scales);
  4. regroup the received source-major rows expert-major (``moe_ep_regroup``), which also writes
     the local expert offsets, and run the grouped FFN over the E_loc local experts;
  5. regroup the FFN output back to source-major order and return it with the reverse all-to-all;
  6. combine: the returned rows sit exactly where the dispatch put the sent ones, so the weighted
     combine uses the dispatch's ``slot_row`` unchanged.

Two exchange modes (the NCCL EP page, section 2.2):
  * ``"ht"`` (high throughput): packed variable-size blocks.  The host reads the send and receive
    sizes once per step (one small device-to-host copy after the count exchange), so a step cannot
    be captured in a CUDA graph.
  * ``"ll"`` (low latency): every (source, destination) block is padded to M = T * min(k, E_loc)
    rows, the most one source can send to one destination, so every all-to-all has equal, fixed
    splits: no host synchronisation, and a whole step can be captured in a CUDA graph.  The padding
    is one more regroup on each side.

A third mode moves the rows over peer memory instead of through all-to-alls (the NCCL EP page,
section 1: kernels that load and store other GPUs' memory over NVLink; section 2.1: the dispatch
delivers each token to its expert owner's buffer and the combine reads the outputs back):
  * ``"p2p"``: the send and return buffers of every rank are mapped into every other rank
    (``comm.alloc_shared``: torch symmetric memory between GPUs).  After the dispatch, one
    all-gather of the [E] counts gives every rank the whole [R, E] count matrix (and orders it after
    every rank's dispatch); ``moe_ep_exchange`` then pulls each rank's rows from the sources' send
    buffers straight into its expert-major FFN input (exchange and regroup in one kernel), and after
    the FFN pushes the outputs straight into the sources' return buffers; a stream-ordered barrier
    later, every rank combines.  No row passes through a staging buffer, no host synchronisation,
    and the step can be captured in a CUDA graph.

Every row of a token meets the same kernels as on a single device: the received rows of expert e
are ordered by (source rank, source token), which is the single-device dispatch order over the
rank-major concatenation of all ranks' tokens, so the FFN and the combine see identical operands,
and the output equals the single-device output bit for bit.

Capacity limits are not applied under expert parallelism (a per-expert limit over all ranks' tokens
needs the counts of every lower rank before the dispatch).  The local steps run through ``ops``
(the CUDA library by default); the exchanges go through ``comm`` (``torch.distributed`` by
default: NCCL between GPUs).
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import _lib
from .layer import expect

A_MAJOR, B_MAJOR = 0, 1


class CudaOps:
    """The local steps of an expert-parallel rank on this GPU: the C-ABI calls of libmoe.so."""

    def __init__(self, device):
        _lib.load()
        self.device = device

    def workspace(self, nbytes):
        return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=self.device)

    def route(self, logits, T, E, k, renormalize, topk_idx, topk_w):
        _lib.moe_route(logits, T, E, k, renormalize, topk_idx, topk_w, None)

    def dispatch(self, x, T, H, topk_idx, k, E, R, payload, send, send_scales, expert_counts,
                 expert_offsets, rank_offsets, slot_row, row_token, ws):
        _lib.moe_dispatch(x, T, H, topk_idx, k, E, R, 0, payload, send, send_scales,
                          expert_counts, expert_offsets, rank_offsets, slot_row, row_token, ws,
                          ws.numel())

    def regroup(self, counts, A, B, src_order, src_stride, src, dst_order, dst_stride, dst,
                src_aux=None, dst_aux=None, dst_offsets=None, status=None):
        _lib.moe_ep_regroup(counts, A, B, src_order, src_stride, src.shape[0], dst_order,
                            dst_stride, dst.shape[0], src, dst, src[0].numel() * src.element_size(),
                            src_aux, dst_aux,
                            0 if src_aux is None else src_aux[0].numel() * src_aux.element_size(),
                            dst_offsets, status)

    def expert_ffn(self, rows, scales, payload, offsets, max_rows, E, H, F, w_gate, w_up, w_down,
                   out, ws):
        _lib.moe_expert_ffn(rows, scales, payload, offsets, max_rows, E, H, F, w_gate, w_up,
                            w_down, out, ws, ws.numel())

    def combine(self, expert_out, max_rows, slot_row, topk_w, T, k, H, y):
        _lib.moe_combine(expert_out, max_rows, slot_row, topk_w, T, k, H, y, None)

    def peer_table(self, tensors):
        return torch.tensor([t.data_ptr() for t in tensors], dtype=torch.int64).to(self.device)

    def exchange(self, all_counts, R, E, rank, direction, peer_rows, peer_aux, peer_cap, local,
                 local_aux, local_offsets=None, status=None):
        _lib.moe_ep_exchange(all_counts, R, E, rank, direction, peer_rows, peer_aux, peer_cap,
                             local, local_aux, local.shape[0],
                             local[0].numel() * local.element_size(),
                             0 if local_aux is None else local_aux[0].numel() * local_aux.element_size(),
                             local_offsets, status)

    def combine_backward(self, dy, T, H, k, E, logits, renormalize, topk_idx, topk_w, slot_row,
                         expert_out, d_eo, d_topk_w, d_logits):
        _lib.moe_combine_backward(dy, T, H, k, E, logits, renormalize, topk_idx, topk_w, slot_row,
                                  expert_out.shape[0], expert_out, d_eo, d_topk_w, d_logits)

    def expert_backward(self, ffn_input, d_eo, offsets, max_rows, E, H, F, w_gate, w_up, w_down,
                        dx_rows, d_w_gate, d_w_up, d_w_down, ws):
        _lib.moe_expert_backward(ffn_input, d_eo, offsets, max_rows, E, H, F, w_gate, w_up, w_down,
                                 dx_rows, d_w_gate, d_w_up, d_w_down, ws, ws.numel())

    def ffn_input_rows(self, rows, scales, payload, ffn_ws, max_rows, H, F):
        """The FFN input rows as bf16 [max_rows, H]: the rows themselves, or, for the FP8 payload,
        the dequantised rows the last expert FFN call left in its workspace (after h)."""
        if payload != _lib.MOE_PAYLOAD_FP8_E4M3_B128:
            return rows
        off = 256 + (max_rows * F * 2 + 255) // 256 * 256
        return ffn_ws[off:off + max_rows * H * 2].view(torch.bfloat16).view(max_rows, H)

    def sync_status(self, ws) -> int:
        return _lib.moe_sync_status(ws)


class TorchComm:
    """The exchange over a ``torch.distributed`` process group (NCCL over NVLink between GPUs;
    gloo on CPU).

    ``all_to_all(out, inp, out_splits, in_splits)`` splits along dim 0 (equal splits when the lists
    are None); ``all_gather(out, inp)`` concatenates every rank's ``inp`` in rank order;
    ``barrier()`` is a one-element all-reduce, ordered on the current stream like any collective;
    ``alloc_shared(shape, dtype, device)`` returns this rank's buffer and every rank's buffer as
    mapped on this GPU (torch symmetric memory; with one rank and ``symmetric`` False, a plain
    allocation)."""

    def __init__(self, group=None, symmetric: bool = False):
        self.group = group
        self.rank = dist.get_rank(group)
        self.size = dist.get_world_size(group)
        self.symmetric = symmetric
        self._handles = []
        self._one = None

    def all_to_all(self, out, inp, out_splits=None, in_splits=None):
        dist.all_to_all_single(out, inp, out_splits, in_splits, group=self.group)

    def all_gather(self, out, inp):
        dist.all_gather_into_tensor(out, inp, group=self.group)

    def barrier(self, device):
        if self._one is None:
            self._one = torch.zeros(1, dtype=torch.int32, device=device)
        dist.all_reduce(self._one, group=self.group)

    def alloc_shared(self, shape, dtype, device):
        if self.size == 1 and not self.symmetric:
            t = torch.empty(shape, dtype=dtype, device=device)
            return t, [t]
        if torch.device(device).type != "cuda":
            raise NotImplementedError("peer buffers need CUDA devices")
        import torch.distributed._symmetric_memory as symm_mem
        t = symm_mem.empty(*shape, dtype=dtype, device=device)
        h = symm_mem.rendezvous(t, self.group if self.group is not None else dist.group.WORLD)
        self._handles.append(h)  # keeps the peer mappings alive
        return t, [h.get_buffer(r, tuple(shape), dtype) for r in range(self.size)]


def _rows_as_bytes(t: torch.Tensor) -> torch.Tensor:
    """A [n, ...] buffer as uint8 [n, row_bytes], so that every backend exchanges it as bytes."""
    return t.view(torch.uint8).view(t.shape[0], -1)


class MoeEP:
    """One expert-parallel MoE layer on this rank: T local tokens of width H, E experts over the
    R ranks of ``comm`` (E % R == 0), top-k, SwiGLU FFN width F.

    ``mode`` is "ht" or "ll" (see the module docstring); ``payload`` is "bf16" or "fp8" (e4m3 codes
    plus one fp32 scale per 128 elements cross the exchange; the FFN output returns in bf16).
    ``recv_rows`` is the initial receive capacity in rows for "ht" (grown when a step needs more;
    default T*k); "ll" always holds R*M rows.  Weights are this rank's experts only:
    ``w_gate``, ``w_up`` [E_loc, F, H] and ``w_down`` [E_loc, H, F], bf16.
    ``comm`` carries the all-to-alls (default: ``TorchComm`` over the default process group).
    """

    def __init__(self, T: int, H: int, E: int, k: int, F: int, comm=None, payload: str = "bf16",
                 mode: str = "ht", renormalize: bool = True, recv_rows: int | None = None,
                 device="cuda", ops=None):
        if mode not in ("ht", "ll", "p2p"):
            raise ValueError("mode must be 'ht', 'll' or 'p2p'")
        if payload not in ("bf16", "fp8"):
            raise ValueError("payload must be 'bf16' or 'fp8'")
        self.comm = TorchComm() if comm is None else comm
        self.R = self.comm.size
        self.rank = self.comm.rank
        if E % self.R != 0:
            raise ValueError(f"E={E} is not a multiple of the {self.R} ranks")
        self.T, self.H, self.E, self.k, self.F = T, H, E, k, F
        self.E_loc = E // self.R
        self.mode = mode
        self.renormalize = bool(renormalize)
        self.fp8 = payload == "fp8"
        self.payload = _lib.MOE_PAYLOAD_FP8_E4M3_B128 if self.fp8 else _lib.MOE_PAYLOAD_BF16
        dev = torch.device(device)
        if dev.type == "cuda" and dev.index is None:
            dev = torch.device("cuda", torch.cuda.current_device())
        self.device = dev
        self.ops = CudaOps(dev) if ops is None else ops
        i32 = dict(dtype=torch.int32, device=dev)
        S = T * k
        self.M = T * min(k, self.E_loc)  # most rows one source sends one destination
        self.row_dtype = torch.uint8 if self.fp8 else torch.bfloat16
        self.nb = H // 128 if self.fp8 else 0  # scale blocks per row
        # local side: route, dispatch, combine on this rank's tokens
        self.topk_idx = torch.empty((T, k), **i32)
        self.topk_w = torch.empty((T, k), dtype=torch.float32, device=dev)
        if mode == "p2p":
            # every rank's send and return buffers, as mapped on this GPU
            self.send, peers = self.comm.alloc_shared((max(S, 1), H), self.row_dtype, dev)
            self.peer_send = self._pointers(peers)
            self.send_scales, self.peer_send_scales = None, None
            if self.fp8:
                self.send_scales, peers = self.comm.alloc_shared((max(S, 1), self.nb),
                                                                 torch.float32, dev)
                self.peer_send_scales = self._pointers(peers)
            self.ret, peers = self.comm.alloc_shared((max(S, 1), H), torch.bfloat16, dev)
            self.peer_ret = self._pointers(peers)
            self.all_counts = torch.empty(self.R * E, **i32)
        else:
            self.send = torch.empty((S, H), dtype=self.row_dtype, device=dev)
            self.send_scales = torch.empty((S, self.nb), dtype=torch.float32, device=dev) \
                if self.fp8 else None
            self.ret = torch.empty((S, H), dtype=torch.bfloat16, device=dev)  # returned rows
        self.expert_counts = torch.empty(E, **i32)
        self.expert_offsets = torch.empty(E + 1, **i32)
        self.rank_offsets = torch.empty(self.R + 1, **i32)
        self.slot_row = torch.empty((T, k), **i32)
        self.row_token = torch.empty(max(S, 1), **i32)
        self.y = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
        self.ws_dispatch = self.ops.workspace(_lib.moe_dispatch_workspace_size(T, E, k))
        # the status word of the regroups (counts from other ranks are checked on the device)
        self.ws_regroup = self.ops.workspace(256)
        # expert side
        self.recv_counts = torch.empty(self.R * self.E_loc, **i32)
        self.local_offsets = torch.empty(self.E_loc + 1, **i32)
        if mode == "p2p":
            self._alloc_expert_side(self.R * self.M)
        elif mode == "ll":
            P = self.R * self.M
            self.send_pad = torch.empty((P, H), dtype=self.row_dtype, device=dev)
            self.send_pad_scales = torch.empty((P, self.nb), dtype=torch.float32, device=dev) \
                if self.fp8 else None
            self.ret_pad = torch.empty((P, H), dtype=torch.bfloat16, device=dev)
            self._alloc_expert_side(P)
        else:
            self._alloc_expert_side(max(int(recv_rows) if recv_rows else S, 1))
            self._sizes = torch.empty(self.R + 1 + self.R * self.E_loc, dtype=torch.int32,
                                      pin_memory=dev.type == "cuda")

    def _alloc_expert_side(self, rows: int):
        dev, H = self.device, self.H
        self.cap = rows
        self.recv = torch.empty((rows, H), dtype=self.row_dtype, device=dev)
        self.recv_scales = torch.empty((rows, self.nb), dtype=torch.float32, device=dev) \
            if self.fp8 else None
        self.grouped = torch.empty((rows, H), dtype=self.row_dtype, device=dev)
        self.grouped_scales = torch.empty((rows, self.nb), dtype=torch.float32, device=dev) \
            if self.fp8 else None
        self.expert_out = torch.empty((rows, H), dtype=torch.bfloat16, device=dev)
        self.back = torch.empty((rows, H), dtype=torch.bfloat16, device=dev)
        self.ws_ffn = self.ops.workspace(
            _lib.moe_ffn_workspace_size(rows, self.E_loc, H, self.F, self.payload))

    def _pointers(self, tensors):
        """The buffers as the exchange step takes them (``ops.peer_table``: for the CUDA library,
        a device array of their addresses, int64 [R])."""
        return self.ops.peer_table(tensors)

    # -- the exchange -------------------------------------------------------------------------
    def _all_to_all(self, out, inp, out_splits=None, in_splits=None):
        self.comm.all_to_all(out, inp, out_splits, in_splits)

    def _exchange_rows(self, out, inp, out_splits, in_splits):
        self._all_to_all(_rows_as_bytes(out), _rows_as_bytes(inp), out_splits, in_splits)

    def _ht_sizes(self):
        """Send and receive row counts per peer: one device-to-host copy after the count exchange."""
        R = self.R
        self._sizes[:R + 1].copy_(self.rank_offsets, non_blocking=True)
        self._sizes[R + 1:].copy_(self.recv_counts, non_blocking=True)
        if self.device.type == "cuda":
            torch.cuda.current_stream(self.device).synchronize()
        ro = self._sizes[:R + 1].tolist()
        rc = self._sizes[R + 1:].view(R, self.E_loc).sum(1).tolist()
        send_splits = [ro[d + 1] - ro[d] for d in range(R)]
        return send_splits, [int(v) for v in rc]

    # -- one step -----------------------------------------------------------------------------
    def forward(self, logits, x, w_gate, w_up, w_down) -> torch.Tensor:
        T, H, E, k, R, E_loc = self.T, self.H, self.E, self.k, self.R, self.E_loc
        dev = self.device
        expect(logits, (T, E), torch.float32, "logits", dev)
        expect(x, (T, H), torch.bfloat16, "x", dev)
        expect(w_gate, (E_loc, self.F, H), torch.bfloat16, "w_gate", dev)
        expect(w_up, (E_loc, self.F, H), torch.bfloat16, "w_up", dev)
        expect(w_down, (E_loc, H, self.F), torch.bfloat16, "w_down", dev)
        ops = self.ops
        ops.route(logits, T, E, k, self.renormalize, self.topk_idx, self.topk_w)
        ops.dispatch(x, T, H, self.topk_idx, k, E, R, self.payload, self.send, self.send_scales,
                     self.expert_counts, self.expert_offsets, self.rank_offsets, self.slot_row,
                     self.row_token, self.ws_dispatch)
        st = self.ws_regroup
        if self.mode == "p2p":
            return self._forward_p2p(w_gate, w_up, w_down, st)
        # counts: expert_counts is [R destinations, E_loc] already
        self._all_to_all(self.recv_counts, self.expert_counts)
        if self.mode == "ht":
            send_splits, recv_splits = self._ht_sizes()
            n_recv = sum(recv_splits)
            if n_recv > self.cap:
                self._alloc_expert_side(max(n_recv, self.cap + self.cap // 4))
            n_send = sum(send_splits)
            self._ht_splits = (send_splits, recv_splits)  # the backward retraces them
            self._exchange_rows(self.recv[:n_recv], self.send[:n_send], recv_splits, send_splits)
            if self.fp8:
                self._all_to_all(self.recv_scales[:n_recv], self.send_scales[:n_send],
                                 recv_splits, send_splits)
            src_stride = 0
        else:
            ops.regroup(self.expert_counts, R, E_loc, A_MAJOR, 0, self.send, A_MAJOR, self.M,
                        self.send_pad, self.send_scales, self.send_pad_scales, None, st)
            self._exchange_rows(self.recv, self.send_pad, None, None)
            if self.fp8:
                self._all_to_all(self.recv_scales, self.send_pad_scales)
            src_stride = self.M
        # expert-major for the grouped FFN; local_offsets are the FFN's expert offsets
        ops.regroup(self.recv_counts, R, E_loc, A_MAJOR, src_stride, self.recv, B_MAJOR, 0,
                    self.grouped, self.recv_scales, self.grouped_scales, self.local_offsets, st)
        ops.expert_ffn(self.grouped, self.grouped_scales, self.payload, self.local_offsets,
                       self.cap, E_loc, H, self.F, w_gate, w_up, w_down, self.expert_out,
                       self.ws_ffn)
        ops.regroup(self.recv_counts, R, E_loc, B_MAJOR, 0, self.expert_out, A_MAJOR, src_stride,
                    self.back, None, None, None, st)
        if self.mode == "ht":
            self._exchange_rows(self.ret[:n_send], self.back[:n_recv], send_splits, recv_splits)
        else:
            self._exchange_rows(self.ret_pad, self.back, None, None)
            ops.regroup(self.expert_counts, R, E_loc, A_MAJOR, self.M, self.ret_pad, A_MAJOR, 0,
                        self.ret, None, None, None, st)
        ops.combine(self.ret, self.ret.shape[0], self.slot_row, self.topk_w, T, k, H, self.y)
        return self.y

    def _forward_p2p(self, w_gate, w_up, w_down, st):
        T, H, E, k, R = self.T, self.H, self.E, self.k, self.R
        ops, S = self.ops, self.send.shape[0]
        # the whole [R, E] count matrix; as a collective it also follows every rank's dispatch
        self.comm.all_gather(self.all_counts, self.expert_counts)
        ops.exchange(self.all_counts, R, E, self.rank, _lib.MOE_EP_PULL, self.peer_send,
                     self.peer_send_scales, S, self.grouped, self.grouped_scales,
                     self.local_offsets, st)
        ops.expert_ffn(self.grouped, self.grouped_scales, self.payload, self.local_offsets,
                       self.cap, self.E_loc, H, self.F, w_gate, w_up, w_down, self.expert_out,
                       self.ws_ffn)
        ops.exchange(self.all_counts, R, E, self.rank, _lib.MOE_EP_PUSH, self.peer_ret, None, S,
                     self.expert_out, None, None, st)
        # every rank's pushes into this rank's return buffer are complete after the barrier
        self.comm.barrier(self.device)
        ops.combine(self.ret, S, self.slot_row, self.topk_w, T, k, H, self.y)
        return self.y

    # -- backward ------------------------------------------------------------------------------
    def _alloc_backward(self):
        dev, H, S = self.device, self.H, self.send.shape[0]
        bf16, f32 = torch.bfloat16, torch.float32
        E_loc, F = self.E_loc, self.F
        if self.mode == "p2p":
            # the experts' ranks pull d_eo from the sources and push dx_rows back into them
            self.b_d_eo, peers = self.comm.alloc_shared((S, H), bf16, dev)
            self.b_peer_d_eo = self._pointers(peers)
            self.b_dret, peers = self.comm.alloc_shared((S, H), bf16, dev)
            self.b_peer_dret = self._pointers(peers)
        else:
            self.b_d_eo = torch.empty((S, H), dtype=bf16, device=dev)
            self.b_dret = torch.empty((S, H), dtype=bf16, device=dev)
            P = self.cap if self.mode == "ht" else self.R * self.M
            self.b_recv = torch.empty((P, H), dtype=bf16, device=dev)      # d_eo, source order
            self.b_back = torch.empty((P, H), dtype=bf16, device=dev)      # dx_rows, source order
            if self.mode == "ll":
                self.b_send_pad = torch.empty((self.R * self.M, H), dtype=bf16, device=dev)
                self.b_ret_pad = torch.empty((self.R * self.M, H), dtype=bf16, device=dev)
        self.b_cap = self.cap
        self.b_d_eo_grouped = torch.empty((self.cap, H), dtype=bf16, device=dev)
        self.b_dx_rows = torch.empty((self.cap, H), dtype=bf16, device=dev)
        self.ws_ebwd = self.ops.workspace(
            _lib.moe_expert_backward_workspace_size(self.cap, F))
        self.ones = torch.ones((self.T, self.k), dtype=f32, device=dev)
        self.grads = {
            "dx": torch.empty((self.T, H), dtype=bf16, device=dev),
            "d_logits": torch.empty((self.T, self.E), dtype=f32, device=dev),
            "d_topk_w": torch.empty((self.T, self.k), dtype=f32, device=dev),
            "d_w_gate": torch.empty((E_loc, F, H), dtype=f32, device=dev),
            "d_w_up": torch.empty((E_loc, F, H), dtype=f32, device=dev),
            "d_w_down": torch.empty((E_loc, H, F), dtype=f32, device=dev),
        }

    def backward(self, dy, logits, w_gate, w_up, w_down) -> dict:
        """Gradients for the output gradient ``dy`` [T,H] bf16 of this rank's tokens, after
        ``forward`` (its routing, plan, exchanged rows and counts are reused): the combine backward
        on this rank (the d_eo rows, the routing-weight and logit gradients), d_eo to the experts'
        owners the way the rows went, the experts' backward there (the weight gradients of this
        rank's experts), dx_rows back the way the outputs came, and the unit-weight combine.
        Returns dx bf16 [T,H], d_logits fp32 [T,E], d_topk_w fp32 [T,k] for this rank's tokens
        and d_w_gate / d_w_up fp32 [E_loc,F,H], d_w_down fp32 [E_loc,H,F] for its experts."""
        T, H, E, k, R, E_loc = self.T, self.H, self.E, self.k, self.R, self.E_loc
        dev = self.device
        expect(dy, (T, H), torch.bfloat16, "dy", dev)
        expect(logits, (T, E), torch.float32, "logits", dev)
        expect(w_gate, (E_loc, self.F, H), torch.bfloat16, "w_gate", dev)
        expect(w_up, (E_loc, self.F, H), torch.bfloat16, "w_up", dev)
        expect(w_down, (E_loc, H, self.F), torch.bfloat16, "w_down", dev)
        if getattr(self, "grads", None) is None or self.b_cap != self.cap:
            self._alloc_backward()
        ops, g, st = self.ops, self.grads, self.ws_regroup
        S = self.send.shape[0]
        ops.combine_backward(dy, T, H, k, E, logits, self.renormalize, self.topk_idx, self.topk_w,
                             self.slot_row, self.ret, self.b_d_eo, g["d_topk_w"], g["d_logits"])
        if self.mode == "p2p":
            self.comm.barrier(dev)  # every rank's d_eo rows are written
            ops.exchange(self.all_counts, R, E, self.rank, _lib.MOE_EP_PULL, self.b_peer_d_eo,
                         None, S, self.b_d_eo_grouped, None, None, st)
        elif self.mode == "ht":
            send_splits, recv_splits = self._ht_splits
            n_send, n_recv = sum(send_splits), sum(recv_splits)
            self._exchange_rows(self.b_recv[:n_recv], self.b_d_eo[:n_send], recv_splits,
                                send_splits)
            ops.regroup(self.recv_counts, R, E_loc, A_MAJOR, 0, self.b_recv, B_MAJOR, 0,
                        self.b_d_eo_grouped, None, None, None, st)
        else:
            ops.regroup(self.expert_counts, R, E_loc, A_MAJOR, 0, self.b_d_eo, A_MAJOR, self.M,
                        self.b_send_pad, None, None, None, st)
            self._exchange_rows(self.b_recv, self.b_send_pad, None, None)
            ops.regroup(self.recv_counts, R, E_loc, A_MAJOR, self.M, self.b_recv, B_MAJOR, 0,
                        self.b_d_eo_grouped, None, None, None, st)
        x_rows = ops.ffn_input_rows(self.grouped, self.grouped_scales, self.payload, self.ws_ffn,
                                    self.cap, H, self.F)
        ops.expert_backward(x_rows, self.b_d_eo_grouped, self.local_offsets, self.cap, E_loc, H,
                            self.F, w_gate, w_up, w_down, self.b_dx_rows, g["d_w_gate"],
                            g["d_w_up"], g["d_w_down"], self.ws_ebwd)
        if self.mode == "p2p":
            ops.exchange(self.all_counts, R, E, self.rank, _lib.MOE_EP_PUSH, self.b_peer_dret,
                         None, S, self.b_dx_rows, None, None, st)
            self.comm.barrier(dev)  # every rank's pushes into this rank's buffer are complete
        elif self.mode == "ht":
            ops.regroup(self.recv_counts, R, E_loc, B_MAJOR, 0, self.b_dx_rows, A_MAJOR, 0,
                        self.b_back, None, None, None, st)
            self._exchange_rows(self.b_dret[:n_send], self.b_back[:n_recv], send_splits,
                                recv_splits)
        else:
            ops.regroup(self.recv_counts, R, E_loc, B_MAJOR, 0, self.b_dx_rows, A_MAJOR, self.M,
                        self.b_back, None, None, None, st)
            self._exchange_rows(self.b_ret_pad, self.b_back, None, None)
            ops.regroup(self.expert_counts, R, E_loc, A_MAJOR, self.M, self.b_ret_pad, A_MAJOR, 0,
                        self.b_dret, None, None, None, st)
        ops.combine(self.b_dret, S, self.slot_row, self.ones, T, k, H, g["dx"])
        return g

    def status(self) -> int:
        """Synchronise; the first non-OK device status of this rank's dispatch, regroups and FFN."""
        for ws in (self.ws_dispatch, self.ws_regroup, self.ws_ffn) + (
                (self.ws_ebwd,) if getattr(self, "ws_ebwd", None) is not None else ()):
            st = self.ops.sync_status(ws)
            if st != _lib.MOE_OK:
                return st
        return _lib.MOE_OK
