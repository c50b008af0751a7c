"""The whole step captured as one CUDA graph: replays match eager calls bit for bit."""
import math

import pytest
import torch

import moe_inputs as mi


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["tiny", "decode-small", "finegrained-small", "skewed-small"])
def test_graph_replay_matches_eager(cuda, name):
    from combine_moe_route_10_b200 import MoeShuffle
    w = mi.get(name)
    cap = math.ceil(w.capacity_factor * w.T * w.k / w.E) if w.capacity_factor else 0
    d0 = mi.make_inputs(w, seed=0, device="cuda")
    d1 = mi.make_inputs(w, seed=1, device="cuda", weights=False)
    wts = (d0["w_gate"], d0["w_up"], d0["w_down"])
    eager = MoeShuffle(w.T, w.H, w.E, w.k, w.R, w.F, payload=w.payload, capacity=cap)
    graphed = MoeShuffle(w.T, w.H, w.E, w.k, w.R, w.F, payload=w.payload, capacity=cap)
    logits = d0["logits"].clone()
    x = d0["x"].clone()
    out = torch.empty_like(graphed.y)
    g = graphed.capture(logits, x, *wts, out=out)
    for d in (d0, d1, d0):
        logits.copy_(d["logits"])
        x.copy_(d["x"])
        g.replay()
        y_ref = eager.forward(d["logits"], d["x"], *wts).clone()
        torch.cuda.synchronize()
        assert torch.equal(out, y_ref)
        assert torch.equal(graphed.y, y_ref)
        assert torch.equal(graphed.slot_row, eager.slot_row)
    assert graphed.status() == 0 and eager.status() == 0
