"""Per-expert weight lists: each expert's weights in its own allocation ("DWDP: 在NVL72上的高性能
分布式权重数据并行", sections 消除D2D时延开销 and 关键优化实施: the grouped GEMM consumes a list of
weight buffers instead of merged [E, ...] arrays).

moe_expert_ffn_list must give exactly moe_expert_ffn's results on the same values (same tiles, same
k order), and the oracle's within the parity bar, for experts of both kernels (a handful of rows,
and several row blocks), ragged F and H, and the FP8 payload."""
import numpy as np
import pytest
import torch

import moe_inputs as mi
from _helpers import assert_ffn_and_combine, bits16, np_
from oracle import moe

pytestmark = pytest.mark.gpu


def split_weights(d, E):
    """Each expert's three matrices copied into separate allocations, with gaps between them."""
    keep = []
    out = {}
    for name in ("w_gate", "w_up", "w_down"):
        ts = []
        for e in range(E):
            keep.append(torch.empty(4096, dtype=torch.uint8, device="cuda"))  # a gap
            ts.append(d[name][e].clone())
        out[name] = ts
    return out, keep


@pytest.mark.parametrize("name", ["tiny", "train-small", "finegrained-small", "skewed-small"])
def test_weight_list_matches_contiguous_weights_and_oracle(cuda, name):
    from combine_moe_route_10_b200 import MoeShuffle
    w = mi.get(name)
    d = mi.make_inputs(w, seed=3, device="cuda")
    cap = moe.capacity(w.capacity_factor, w.T, w.k, w.E)
    m = MoeShuffle(w.T, w.H, w.E, w.k, w.R, w.F, payload=w.payload, capacity=cap)
    y_ref = m.forward(d["logits"], d["x"], d["w_gate"], d["w_up"], d["w_down"]).clone()
    h_ref, eo_ref = m.h.clone(), m.expert_out.clone()
    assert m.status() == 0
    parts, _keep = split_weights(d, w.E)
    wlist = m.expert_weight_list(parts["w_gate"], parts["w_up"], parts["w_down"])
    for _ in range(2):          # twice in a row: the workspace counters reset inside each call
        m.expert_out.zero_()
        m.expert_ffn_list(wlist)
        m.combine()
        assert m.status() == 0
        S = int(m.expert_offsets[w.E].item())
        assert torch.equal(m.h[:S], h_ref[:S])
        assert torch.equal(m.expert_out[:S], eo_ref[:S])
        assert torch.equal(m.y, y_ref)
    o = moe.pipeline(np_(d["logits"]), bits16(d["x"]), bits16(d["w_gate"]), bits16(d["w_up"]),
                     bits16(d["w_down"]), w.k, w.R, w.capacity_factor, w.payload == "fp8")
    assert_ffn_and_combine(bits16(m.h)[:S], bits16(m.expert_out)[:S], bits16(m.y), o["h"],
                           o["expert_out"], o["y"], o["expert_offsets"], d["w_down"],
                           o["slot_row"], o["topk_w"], name)


@pytest.mark.parametrize("rows,H,F", [([40, 300, 0, 129], 320, 192),    # ragged H and F
                                      ([1, 64, 65, 500], 256, 320)])
def test_weight_list_edge_shapes(cuda, rows, H, F):
    from combine_moe_route_10_b200 import MoeShuffle
    E = len(rows)
    off = np.concatenate([[0], np.cumsum(rows)]).astype(np.int32)
    S = int(off[-1])
    g = torch.Generator(device="cuda").manual_seed(S)
    x = mi.randn_bf16((S, H), g)
    d = {"w_gate": mi.randn_bf16((E, F, H), g, 0.05), "w_up": mi.randn_bf16((E, F, H), g, 0.05),
         "w_down": mi.randn_bf16((E, H, F), g, 0.05)}
    m = MoeShuffle(S, H, E, 1, 1, F)
    offd = torch.from_numpy(off).cuda()
    m.expert_ffn(d["w_gate"], d["w_up"], d["w_down"], send=x, expert_offsets=offd)
    eo_ref = m.expert_out[:S].clone()
    parts, _keep = split_weights(d, E)
    wlist = m.expert_weight_list(parts["w_gate"], parts["w_up"], parts["w_down"])
    m.expert_out.zero_()
    m.expert_ffn_list(wlist, send=x, expert_offsets=offd)
    assert m.status() == 0
    assert torch.equal(m.expert_out[:S], eo_ref)
