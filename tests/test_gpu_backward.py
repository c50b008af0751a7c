"""The backward pass on the GPU through the C ABI (``moe_backward``) against the oracle's backward.

The oracle is given the GPU forward's own routing, plan, FFN input rows and expert outputs, so the
comparison covers the backward kernels alone: d_eo bit-exact (one fp32 product, one bf16 rounding),
the unit-weight combine of dx_rows bit-exact, the recomputed h, dg, du, dx_rows and dx within the
bf16 parity bar, the fp32 weight gradients, routing-weight and logit gradients within 1e-2 of the
largest element.  Workloads: every small one (ragged F and H tails, the FP8 payload, capacity drops,
E = 256 with k = 8), both weight modes, and an expert with no rows.
"""
import numpy as np
import pytest
import torch

import moe_inputs as mi
from _helpers import (assert_close_bf16, bf16_values as bf16_vals, bits16, combine_magnitude,
                      combine_row_atol, ffn_row_atol, np_)
from oracle.numerics import bf16_bits as bits_of
from oracle import moe

pytestmark = pytest.mark.gpu


def _rel_max(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.max(np.abs(got - ref)) / max(np.max(np.abs(ref)), 1e-30))


def _run(name, renormalize=True, seed=11, zero_expert=None):
    from combine_moe_route_10_b200 import MoeShuffle
    w = mi.get(name)
    d = mi.make_inputs(w, seed=seed, device="cuda")
    if zero_expert is not None:
        d["logits"][:, zero_expert] = -1e4  # nobody routes here: an expert without rows
    cap = moe.capacity(w.capacity_factor, w.T, w.k, w.E)
    m = MoeShuffle(w.T, w.H, w.E, w.k, w.R, w.F, payload=w.payload, capacity=cap,
                   renormalize=renormalize)
    m.forward(d["logits"], d["x"], d["w_gate"], d["w_up"], d["w_down"])
    g = torch.Generator(device="cuda").manual_seed(seed + 1)
    dy = torch.randn((w.T, w.H), generator=g, device="cuda").to(torch.bfloat16)
    grads = m.backward(dy, d["logits"], d["w_gate"], d["w_up"], d["w_down"])
    torch.cuda.synchronize()
    assert m.status() == 0
    fp8 = w.payload == "fp8"
    S = int(m.expert_offsets[w.E].item())
    fwd = {"slot_row": np_(m.slot_row), "topk_w": np_(m.topk_w), "topk_idx": np_(m.topk_idx),
           "expert_offsets": np_(m.expert_offsets), "expert_out": bits16(m.expert_out)[:S]}
    if fp8:
        fwd["send"] = np_(m.send.view(torch.uint8))[:S]
        fwd["send_scales"] = np_(m.send_scales)[:S]
    else:
        fwd["send"] = bits16(m.send)[:S]
        fwd["send_scales"] = None
    ref = moe.backward(fwd, bits16(dy), np_(d["logits"]), bits16(d["w_gate"]), bits16(d["w_up"]),
                       bits16(d["w_down"]), renormalize=renormalize, fp8=fp8)
    return w, m, d, grads, ref, S


def _check(w, m, m_w, grads, ref, S, what):
    # 1. combine backward: one fp32 product and one bf16 rounding per element
    assert np.array_equal(bits16(m.backward_intermediate("d_eo"))[:S], ref["d_eo"]), what
    # 2. expert backward (fp32 accumulation on the tensor cores against fp64)
    # the recomputed h against the forward's h (itself held to the oracle by the FFN tests)
    assert_close_bf16(bits16(m.backward_intermediate("h"))[:S], bits16(m.h)[:S], f"{what} h")
    for key in ("dg", "du"):
        assert_close_bf16(bits16(m.backward_intermediate(key))[:S], ref[key], f"{what} {key}")
    # dx_rows = dg Wg + du Wu: a one-ulp flip of a bf16 dg or du (fp32 against fp64 before the
    # rounding) moves it by ulp * |W|, the same allowance as the forward's expert_out for h flips
    dg_du = np.maximum(np.abs(bf16_vals(ref["dg"])), np.abs(bf16_vals(ref["du"])))
    w_gu = torch.maximum(m_w["w_gate"].abs(), m_w["w_up"].abs())
    dxr_atol = ffn_row_atol(bits_of(dg_du), np_(m.expert_offsets), w_gu)
    assert_close_bf16(bits16(m.backward_intermediate("dx_rows"))[:S], ref["dx_rows"],
                      f"{what} dx_rows", row_atol=dxr_atol)
    # 3. dx: the unit-weight combine of the GPU's own dx_rows is bit-exact
    dx_rows = bits16(m.backward_intermediate("dx_rows"))
    comb = moe.combine(dx_rows, np_(m.slot_row), np.ones((w.T, w.k), np.float32), w.T, w.H)
    assert np.array_equal(bits16(grads["dx"]), comb), what
    # dx sums k rows that may cancel: its elements are held to the size of their summands, as
    # the forward's combine output is
    ones = np.ones((w.T, w.k), np.float32)
    assert_close_bf16(bits16(grads["dx"]), ref["dx"], f"{what} dx",
                      combine_magnitude(ref["dx_rows"], np_(m.slot_row), ones),
                      combine_row_atol(ref["dx_rows"], np_(m.slot_row), ones, dxr_atol))
    # 4. fp32 gradients
    for key in ("d_w_gate", "d_w_up", "d_w_down"):
        assert _rel_max(np_(grads[key]), ref[key]) <= 1e-2, (what, key)
    assert _rel_max(np_(grads["d_topk_w"]), ref["d_w"]) <= 1e-2, what
    assert _rel_max(np_(grads["d_logits"]), ref["d_logits"]) <= 1e-2, what


@pytest.mark.parametrize("name", ["tiny", "decode-small", "train-small", "skewed-small",
                                  "finegrained-small"])
def test_backward_matches_oracle(cuda, name):
    w, m, d, grads, ref, S = _run(name)
    _check(w, m, d, grads, ref, S, name)


def test_backward_full_softmax_weights(cuda):
    w, m, d, grads, ref, S = _run("train-small", renormalize=False)
    _check(w, m, d, grads, ref, S, "train-small full softmax")


def test_backward_expert_without_rows_gets_zero_weight_gradients(cuda):
    w, m, d, grads, ref, S = _run("tiny", zero_expert=3)
    assert int(m.expert_counts[3].item()) == 0
    for key in ("d_w_gate", "d_w_up", "d_w_down"):
        assert float(grads[key][3].abs().max().item()) == 0.0, key
    _check(w, m, d, grads, ref, S, "tiny, expert 3 idle")


def _sub_problem(m, w, e, S):
    """The forward restricted to expert e's rows: its tokens' slots that landed in e (the others
    dropped), expert offsets [0, n], as the oracle's backward takes them."""
    off = np_(m.expert_offsets)
    lo, hi = int(off[e]), int(off[e + 1])
    sr = np_(m.slot_row).astype(np.int64)
    keep = (sr >= lo) & (sr < hi)
    toks = np.unique(np.nonzero(keep)[0])
    sub_sr = np.where(keep[toks], sr[toks] - lo, -1).astype(np.int32)
    return lo, hi, toks, sub_sr


@pytest.mark.parametrize("name", ["train", "skewed", "finegrained"])
def test_backward_full_size(cuda, name):
    """Full size, as the benchmark runs it: d_eo bit-exact on every row, d_topk_w and d_logits on
    every token, dx bit-exact against the unit-weight combine of the GPU's dx_rows on every token,
    and for two whole experts (the smallest and the largest of at most 1024 rows) the oracle's
    backward on their rows: dg, du, dx_rows and the three weight-gradient matrices."""
    from combine_moe_route_10_b200 import MoeShuffle
    w = mi.get(name)
    d = mi.make_inputs(w, seed=0, device="cuda")
    cap = moe.capacity(w.capacity_factor, w.T, w.k, w.E)
    m = MoeShuffle(w.T, w.H, w.E, w.k, w.R, w.F, payload=w.payload, capacity=cap)
    m.forward(d["logits"], d["x"], d["w_gate"], d["w_up"], d["w_down"])
    g = torch.Generator(device="cuda").manual_seed(5)
    dy = torch.randn((w.T, w.H), generator=g, device="cuda").to(torch.bfloat16)
    grads = m.backward(dy, d["logits"], d["w_gate"], d["w_up"], d["w_down"])
    torch.cuda.synchronize()
    assert m.status() == 0
    fp8 = w.payload == "fp8"
    S = int(m.expert_offsets[w.E].item())
    sr = np_(m.slot_row).astype(np.int64)
    tw = np_(m.topk_w)
    dyf = np_(dy.float())
    eo = np_(m.expert_out[:S].float()).astype(np.float64)
    # every row: d_eo = bf16(fp32(w) * fp32(dy)); every slot: d_w = <dy, eo>
    d_eo = bits16(m.backward_intermediate("d_eo"))[:S]
    d_w_ref = np.zeros(sr.shape)
    for j in range(w.k):
        ok = sr[:, j] >= 0
        rows = sr[ok, j]
        prod = (tw[ok, j][:, None].astype(np.float32) * dyf[ok]).astype(np.float32)
        assert np.array_equal(d_eo[rows], bits_of(prod.astype(np.float64))), (name, j)
        d_w_ref[ok, j] = np.einsum("th,th->t", dyf[ok].astype(np.float64), eo[rows])
    assert _rel_max(np_(grads["d_topk_w"]), d_w_ref) <= 1e-2, name
    # d_logits from d_w (renormalised top-k softmax)
    idx = np_(m.topk_idx).astype(np.int64)
    dl_ref = np.zeros((w.T, w.E))
    c = np.sum(tw * d_w_ref, axis=1)
    np.put_along_axis(dl_ref, idx, tw * (d_w_ref - c[:, None]), axis=1)
    assert _rel_max(np_(grads["d_logits"]), dl_ref) <= 1e-2, name
    # dx: the unit-weight combine of the GPU's dx_rows, every token
    dx_rows = bits16(m.backward_intermediate("dx_rows"))
    comb = moe.combine(dx_rows, np_(m.slot_row), np.ones((w.T, w.k), np.float32), w.T, w.H)
    assert np.array_equal(bits16(grads["dx"]), comb), name
    # two whole experts through the oracle
    counts = np.diff(np_(m.expert_offsets))
    nz = np.nonzero(counts)[0]
    small = int(nz[np.argmin(counts[nz])])
    big_c = [e for e in nz if counts[e] <= 1024]
    big = int(max(big_c, key=lambda e: counts[e]))
    wb = [bits16(d[k_]) for k_ in ("w_gate", "w_up", "w_down")]
    send_rows = (np_(m.send.view(torch.uint8)) if fp8 else bits16(m.send))
    for e in sorted({small, big}):
        lo, hi, toks, sub_sr = _sub_problem(m, w, e, S)
        fwd = {"slot_row": sub_sr, "topk_w": tw[toks], "topk_idx": idx[toks].astype(np.int32),
               "expert_offsets": np.array([0, hi - lo]), "expert_out": bits16(m.expert_out)[lo:hi],
               "send": send_rows[lo:hi],
               "send_scales": np_(m.send_scales)[lo:hi] if fp8 else None}
        ref = moe.backward(fwd, bits16(dy)[toks], np_(d["logits"])[toks], wb[0][e:e + 1],
                           wb[1][e:e + 1], wb[2][e:e + 1], fp8=fp8)
        what = f"{name} expert {e} ({hi - lo} rows)"
        assert np.array_equal(d_eo[lo:hi], ref["d_eo"]), what
        for key in ("dg", "du"):
            assert_close_bf16(bits16(m.backward_intermediate(key))[lo:hi], ref[key], f"{what} {key}")
        dg_du = np.maximum(np.abs(bf16_vals(ref["dg"])), np.abs(bf16_vals(ref["du"])))
        w_gu = torch.maximum(d["w_gate"][e:e + 1].abs(), d["w_up"][e:e + 1].abs())
        dxr_atol = ffn_row_atol(bits_of(dg_du), np.array([0, hi - lo]), w_gu)
        assert_close_bf16(dx_rows[lo:hi], ref["dx_rows"], f"{what} dx_rows", row_atol=dxr_atol)
        for key in ("d_w_gate", "d_w_up", "d_w_down"):
            assert _rel_max(np_(grads[key][e]), ref[key][0]) <= 1e-2, (what, key)


def test_training_step_graph_replays_the_eager_step(cuda):
    """forward + backward captured as one CUDA graph: a replay on new inputs written into the
    captured tensors gives exactly the eager step's outputs and gradients."""
    from combine_moe_route_10_b200 import MoeShuffle
    w = mi.get("train-small")
    d = mi.make_inputs(w, seed=21, device="cuda")
    d2 = mi.make_inputs(w, seed=22, device="cuda", weights=False)
    g = torch.Generator(device="cuda").manual_seed(23)
    dy = torch.randn((w.T, w.H), generator=g, device="cuda").to(torch.bfloat16)
    dy2 = torch.randn((w.T, w.H), generator=g, device="cuda").to(torch.bfloat16)
    # eager reference on the second inputs
    ref = MoeShuffle(w.T, w.H, w.E, w.k, w.R, w.F)
    y_ref = ref.forward(d2["logits"], d2["x"], d["w_gate"], d["w_up"], d["w_down"]).clone()
    g_ref = {k_: v.clone() for k_, v in
             ref.backward(dy2, d2["logits"], d["w_gate"], d["w_up"], d["w_down"]).items()}
    m = MoeShuffle(w.T, w.H, w.E, w.k, w.R, w.F)
    logits, x, dyb = d["logits"].clone(), d["x"].clone(), dy.clone()
    graph = m.capture_step(logits, x, d["w_gate"], d["w_up"], d["w_down"], dyb)
    logits.copy_(d2["logits"])
    x.copy_(d2["x"])
    dyb.copy_(dy2)
    graph.replay()
    torch.cuda.synchronize()
    assert m.status() == 0
    assert torch.equal(m.y, y_ref)
    for key, v in g_ref.items():
        assert torch.equal(m.grads[key], v), key


@pytest.mark.parametrize("T,H,E,k,R,F,payload,cf", [
    (0, 128, 4, 2, 2, 128, "bf16", 0.0),      # empty batch
    (1, 128, 1, 1, 1, 128, "bf16", 0.0),      # one token, one expert
    (3, 64, 2, 2, 1, 64, "bf16", 0.0),        # 6 rows in all, one k-block
    (5, 256, 4, 1, 2, 192, "fp8", 0.0),       # FP8 payload, tiny T, F not a multiple of 128
    (64, 320, 16, 4, 4, 64, "bf16", 1.0),     # H not a multiple of 256, drops at capacity 16
    (200, 192, 8, 8, 8, 128, "bf16", 0.0),    # k = E
    (64, 128, 1024, 32, 32, 64, "bf16", 0.0),  # E and k at their limits: ~2 rows per expert
    (300, 128, 8, 2, 2, 64, "bf16", 0.01),    # capacity 1: almost every slot dropped
])
def test_backward_edge_shapes(cuda, T, H, E, k, R, F, payload, cf):
    from combine_moe_route_10_b200 import MoeShuffle
    w = mi.Workload("edge", T, H, E, k, R, F, payload=payload, capacity_factor=cf)
    d = mi.make_inputs(w, seed=31, device="cuda")
    cap = moe.capacity(cf, T, k, E)
    m = MoeShuffle(T, H, E, k, R, F, payload=payload, capacity=cap)
    m.forward(d["logits"], d["x"], d["w_gate"], d["w_up"], d["w_down"])
    g = torch.Generator(device="cuda").manual_seed(32)
    dy = torch.randn((T, H), generator=g, device="cuda").to(torch.bfloat16)
    grads = m.backward(dy, d["logits"], d["w_gate"], d["w_up"], d["w_down"])
    torch.cuda.synchronize()
    assert m.status() == 0
    if T == 0:
        for key in ("d_w_gate", "d_w_up", "d_w_down"):
            assert float(grads[key].abs().max().item()) == 0.0, key
        return
    fp8 = payload == "fp8"
    S = int(m.expert_offsets[E].item())
    fwd = {"slot_row": np_(m.slot_row), "topk_w": np_(m.topk_w), "topk_idx": np_(m.topk_idx),
           "expert_offsets": np_(m.expert_offsets), "expert_out": bits16(m.expert_out)[:S],
           "send": np_(m.send.view(torch.uint8))[:S] if fp8 else bits16(m.send)[:S],
           "send_scales": np_(m.send_scales)[:S] if fp8 else None}
    ref = moe.backward(fwd, bits16(dy), np_(d["logits"]), bits16(d["w_gate"]), bits16(d["w_up"]),
                       bits16(d["w_down"]), fp8=fp8)
    if cf:
        assert (np_(m.slot_row) < 0).any()
    _check(w, m, d, grads, ref, S, f"edge T{T} E{E} k{k}")


@pytest.mark.parametrize("renormalize", [True, False])
def test_combine_backward_skips_expert_ids_outside_range(cuda, renormalize):
    """An expert id outside [0, E) in one slot (which the forward's dispatch rejects): the combine
    backward's d_eo and d_topk_w do not depend on ids and stay the same; in d_logits the slot adds
    no entry, and every entry of the other slots and tokens is unchanged."""
    from combine_moe_route_10_b200 import MoeShuffle, _lib
    w = mi.get("tiny")
    d = mi.make_inputs(w, seed=4, device="cuda")
    m = MoeShuffle(w.T, w.H, w.E, w.k, w.R, w.F, renormalize=renormalize)
    m.forward(d["logits"], d["x"], d["w_gate"], d["w_up"], d["w_down"])
    g = torch.Generator(device="cuda").manual_seed(9)
    dy = torch.randn((w.T, w.H), generator=g, device="cuda").to(torch.bfloat16)
    idx_bad = m.topk_idx.clone()
    t, j = 3, 1
    e_dropped = int(idx_bad[t, j].item())
    idx_bad[t, j] = w.E + 5

    def run(idx):
        d_eo = torch.zeros((m.max_rows, w.H), dtype=torch.bfloat16, device="cuda")
        d_w = torch.zeros((w.T, w.k), dtype=torch.float32, device="cuda")
        d_lg = torch.full((w.T, w.E), 123.0, dtype=torch.float32, device="cuda")
        _lib.moe_combine_backward(dy, w.T, w.H, w.k, w.E, d["logits"], renormalize, idx,
                                  m.topk_w, m.slot_row, m.max_rows, m.expert_out, d_eo, d_w, d_lg)
        torch.cuda.synchronize()
        return d_eo, d_w, d_lg

    eo_ok, dw_ok, lg_ok = run(m.topk_idx)
    eo_bad, dw_bad, lg_bad = run(idx_bad)
    assert torch.equal(eo_bad, eo_ok) and torch.equal(dw_bad, dw_ok)
    others = [r for r in range(w.T) if r != t]
    assert torch.equal(lg_bad[others], lg_ok[others])
    if renormalize:
        # the other slots keep their entries (c sums over every slot's w d_w, ids aside); the
        # dropped slot's expert, chosen by no other slot of the token, now reads 0
        assert bool((m.topk_idx[t] == e_dropped).sum() == 1)
        expect = lg_ok[t].clone()
        expect[e_dropped] = 0.0
        assert torch.equal(lg_bad[t], expect)
    else:
        assert torch.isfinite(lg_bad[t]).all()
