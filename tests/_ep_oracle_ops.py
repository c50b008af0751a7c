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

    def combine_backward(self, dy, T, H, k, E, logits, renormalize, topk_idx, topk_w, slot_row,
                         expert_out, d_eo, d_topk_w, d_logits):
        self.calls.append("combine_backward")
        S = expert_out.shape[0]
        eo = moe.bf16_from_bits(_u16(expert_out)).astype(np.float64)
        de, dw = moe.combine_backward(_u16(dy), slot_row.numpy(), topk_w.numpy(), eo, S)
        sr = slot_row.numpy()
        rows = sr[sr >= 0]
        _u16(d_eo)[rows] = moe.bf16_bits(de[rows])
        d_topk_w.copy_(torch.from_numpy(dw.astype(np.float32)))
        dl = moe.router_backward(logits.numpy(), topk_idx.numpy(), topk_w.numpy(), dw, renormalize)
        d_logits.copy_(torch.from_numpy(dl.astype(np.float32)))

    def expert_backward(self, ffn_input, d_eo, offsets, max_rows, E, H, F, w_gate, w_up, w_down,
                        dx_rows, d_w_gate, d_w_up, d_w_down, ws):
        self.calls.append("expert_backward")
        off = offsets.numpy().astype(np.int64)
        S = int(off[E])
        xin = moe.bf16_from_bits(_u16(ffn_input)[:S]).astype(np.float64)
        de = moe.bf16_from_bits(_u16(d_eo)[:S]).astype(np.float64)
        r = moe.expert_backward(xin, de, off, _u16(w_gate), _u16(w_up), _u16(w_down))
        _u16(dx_rows)[:S] = moe.bf16_bits(r["dx_rows"])
        d_w_gate.copy_(torch.from_numpy(r["d_w_gate"].astype(np.float32)))
        d_w_up.copy_(torch.from_numpy(r["d_w_up"].astype(np.float32)))
        d_w_down.copy_(torch.from_numpy(r["d_w_down"].astype(np.float32)))

    def ffn_input_rows(self, rows, scales, payload, ffn_ws, max_rows, H, F):
        if payload != 1:
            return rows
        # the FP8 payload's FFN input: the dequantised rows as bf16 (rows past the received ones
        # hold whatever the buffer held; they are never read)
        with np.errstate(over="ignore", invalid="ignore"):
            vals = moe.ffn_inputs(rows.numpy(), scales.numpy(), True)
        out = torch.empty((max_rows, H), dtype=torch.bfloat16)
        _u16(out)[:] = moe.bf16_bits(vals)
        return out

    def sync_status(self, ws) -> int:
        return 0
