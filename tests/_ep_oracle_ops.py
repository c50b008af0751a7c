"""Oracle-backed local steps for ``MoeEP`` on CPU tensors (test infrastructure).

``MoeEP`` runs its local steps through an ``ops`` object (the CUDA library in the product).  These
ops compute the same steps with the oracle, so that the expert-parallel exchange logic (count
exchange, split sizes, padding, regrouping order, return trip) runs for real over gloo ranks on
CPU.  Every buffer is a CPU torch tensor; numpy views write into it in place.
"""
import numpy as np
import torch

from oracle import moe


def _u16(t):
    return t.view(torch.int16).numpy().view(np.uint16)


def _bytes(t):
    return t.view(torch.uint8).numpy().reshape(t.shape[0], -1)


class OracleOps:
    def __init__(self):
        self.device = torch.device("cpu")
        self.calls = []

    def workspace(self, nbytes):
        return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8)

    def route(self, logits, T, E, k, renormalize, topk_idx, topk_w):
        self.calls.append("route")
        idx, w, _ = moe.route(logits.numpy(), k, renormalize)
        topk_idx.copy_(torch.from_numpy(idx.astype(np.int32)))
        topk_w.copy_(torch.from_numpy(w))

    def dispatch(self, x, T, H, topk_idx, k, E, R, payload, send, send_scales, expert_counts,
                 expert_offsets, rank_offsets, slot_row, row_token, ws):
        self.calls.append("dispatch")
        plan = moe.dispatch_plan(topk_idx.numpy(), E, R, 0)
        rows, scales = moe.dispatch_payload(_u16(x), plan, fp8=payload == 1)
        S = plan["S"]
        if payload == 1:
            send.numpy()[:S] = rows
            send_scales.numpy()[:S] = scales
        else:
            _u16(send)[:S] = rows
        expert_counts.copy_(torch.from_numpy(plan["expert_counts"]))
        expert_offsets.copy_(torch.from_numpy(plan["expert_offsets"]))
        rank_offsets.copy_(torch.from_numpy(plan["rank_offsets"]))
        slot_row.copy_(torch.from_numpy(plan["slot_row"]))
        row_token.numpy()[:S] = plan["row_token"]

    def regroup(self, counts, A, B, src_order, src_stride, src, dst_order, dst_stride, dst,
                src_aux=None, dst_aux=None, dst_offsets=None, status=None):
        self.calls.append("regroup")
        c = counts.numpy().reshape(A, B)
        _, off = moe.ep_regroup(c, _bytes(src), src_order, src_stride, _bytes(dst), dst_order,
                                dst_stride)
        if src_aux is not None:
            moe.ep_regroup(c, _bytes(src_aux), src_order, src_stride, _bytes(dst_aux), dst_order,
                           dst_stride)
        if dst_offsets is not None:
            dst_offsets.copy_(torch.from_numpy(off.astype(np.int32)))

    def peer_table(self, tensors):
        return list(tensors)

    def exchange(self, all_counts, R, E, rank, direction, peer_rows, peer_aux, peer_cap, local,
                 local_aux, local_offsets=None, status=None):
        """Peer-memory exchange on CPU: ``peer_rows`` / ``peer_aux`` are the ranks' tensors."""
        self.calls.append("exchange")
        E_loc = E // R
        C = all_counts.numpy().reshape(R, E).astype(np.int64)
        mine = C[:, rank * E_loc:(rank + 1) * E_loc]
        starts = [int(C[s, :rank * E_loc].sum()) for s in range(R)]
        lens = [int(mine[s].sum()) for s in range(R)]
        n = sum(lens)
        for peers, loc in ((peer_rows, local), (peer_aux, local_aux)):
            if peers is None or loc is None:
                continue
            lb = _bytes(loc)
            if direction == 0:      # pull: sources' blocks, source-major, then expert-major
                blocks = np.concatenate([_bytes(peers[s])[starts[s]:starts[s] + lens[s]]
                                         for s in range(R)], axis=0)
                grouped, off = moe.ep_regroup(mine, blocks, 0, 0, np.zeros_like(blocks), 1, 0)
                lb[:n] = grouped
                if local_offsets is not None and loc is local:
                    local_offsets.copy_(torch.from_numpy(off.astype(np.int32)))
            else:                   # push: expert-major back to source-major, into the sources
                back, _ = moe.ep_regroup(mine, lb[:n], 1, 0, np.zeros_like(lb[:n]), 0, 0)
                pos = 0
                for s in range(R):
                    _bytes(peers[s])[starts[s]:starts[s] + lens[s]] = back[pos:pos + lens[s]]
                    pos += lens[s]

    def expert_ffn(self, rows, scales, payload, offsets, max_rows, E, H, F, w_gate, w_up, w_down,
                   out, ws):
        self.calls.append("expert_ffn")
        off = offsets.numpy().astype(np.int64)
        S = int(off[E])
        fp8 = payload == 1
        xin = moe.ffn_inputs(rows.numpy()[:S] if fp8 else _u16(rows)[:S],
                             scales.numpy()[:S] if fp8 else None, fp8)
        _, y = moe.expert_ffn(xin, off, _u16(w_gate), _u16(w_up), _u16(w_down))
        _u16(out)[:S] = y

    def combine(self, expert_out, max_rows, slot_row, topk_w, T, k, H, y):
        self.calls.append("combine")
        _u16(y)[:] = moe.combine(_u16(expert_out), slot_row.numpy(), topk_w.numpy(), T, H)

    def sync_status(self, ws) -> int:
        return 0
