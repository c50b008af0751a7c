"""The seeded synthetic inputs shared by the oracle, the tests and the benchmark: determinism, shapes,
dtypes and the stated recipe (distributions, router biases, the skewed workload's hot expert)."""
import math

import numpy as np
import torch

import moe_inputs as mi
from oracle import moe


def test_same_seed_same_inputs_other_seed_other_inputs():
    w = mi.get("decode-small")
    a = mi.make_inputs(w, seed=0)
    b = mi.make_inputs(w, seed=0)
    c = mi.make_inputs(w, seed=1)
    for key in ("logits", "x", "w_gate", "w_up", "w_down"):
        assert torch.equal(a[key], b[key]), key
        assert not torch.equal(a[key], c[key]), key
    # leaving the weights out does not change the routing inputs
    d = mi.make_inputs(w, seed=0, weights=False)
    assert torch.equal(d["logits"], a["logits"]) and torch.equal(d["x"], a["x"])


def test_shapes_and_dtypes_of_every_workload():
    for name, w in mi.WORKLOADS.items():
        d = mi.make_inputs(w, seed=0, weights=False)
        assert d["logits"].shape == (w.T, w.E) and d["logits"].dtype == torch.float32, name
        assert d["x"].shape == (w.T, w.H) and d["x"].dtype == torch.bfloat16, name
        assert w.E % w.R == 0 and 1 <= w.k <= w.E, name
        if w.payload == "fp8":
            assert w.H % 128 == 0, name
        assert w.H % 64 == 0 and w.F % 64 == 0, name
    w = mi.get("tiny")
    d = mi.make_inputs(w, seed=0)
    assert d["w_gate"].shape == (w.E, w.F, w.H) and d["w_up"].shape == (w.E, w.F, w.H)
    assert d["w_down"].shape == (w.E, w.H, w.F)
    assert all(d[k].dtype == torch.bfloat16 for k in ("w_gate", "w_up", "w_down"))


def test_distributions():
    w = mi.Workload("dist", 4096, 1024, 8, 2, 8, 512)
    d = mi.make_inputs(w, seed=3)
    x = d["x"].float()
    assert abs(x.mean().item()) < 0.01 and abs(x.std().item() - 1.0) < 0.01
    lg = d["logits"]
    assert abs(lg.mean().item()) < 0.01 and abs(lg.std().item() - 1.0) < 0.01
    wg = d["w_gate"].float()
    assert abs(wg.std().item() - 0.02) < 0.0005 and abs(wg.mean().item()) < 0.0005
    # bf16 values are the round-to-nearest-even images of fp32 draws: at most half a bf16 ulp away
    g = torch.Generator().manual_seed(5)
    f = torch.randn(1000, generator=g)
    g = torch.Generator().manual_seed(5)
    b = mi.randn_bf16(1000, g).float()
    assert torch.all((b - f).abs() <= f.abs() * 2.0 ** -8)


def test_router_biases():
    # zipf1.2: ln p of a seeded permutation of p_i ~ i^-1.2, centred
    b = mi.zipf_log_bias(256, 1.2, torch.Generator().manual_seed(0)).double()
    assert abs(b.mean().item()) < 1e-6
    p = np.sort(np.exp(b.numpy() - b.numpy().max()))[::-1]
    ratios = p[0] / p[1:10]
    assert np.allclose(ratios, np.arange(2, 11) ** 1.2, rtol=1e-5)
    # hot0+3 adds exactly 3.0 to expert 0's logits and nothing elsewhere
    w = mi.get("skewed-small")
    biased = mi.make_inputs(w, seed=0, weights=False)["logits"]
    gen = torch.Generator().manual_seed(0)
    plain = torch.randn((w.T, w.E), generator=gen, dtype=torch.float32)
    bias = torch.zeros(w.E)
    bias[0] = 3.0
    assert torch.equal(biased, plain + bias[None, :])
    # normal0.5: one draw per expert, added to every token's logits
    w = mi.get("train-small")
    lg = mi.make_inputs(w, seed=0, weights=False)["logits"]
    gen = torch.Generator().manual_seed(0)
    plain = torch.randn((w.T, w.E), generator=gen, dtype=torch.float32)
    delta = lg - plain
    assert torch.allclose(delta, delta[0:1].expand_as(delta), atol=1e-6)
    assert 0.0 < delta[0].abs().max().item() < 2.5


def test_skewed_workload_hot_expert_share_and_capacity():
    w = mi.get("skewed")
    d = mi.make_inputs(w, seed=0, weights=False)
    idx, _, _ = moe.route(d["logits"].numpy(), w.k)
    share = float((idx == 0).sum()) / idx.size
    assert 0.33 < share < 0.43            # ~38% of routes with +3.0 on expert 0
    assert moe.capacity(w.capacity_factor, w.T, w.k, w.E) == 320 == math.ceil(1.25 * 16384 * 2 / 128)
