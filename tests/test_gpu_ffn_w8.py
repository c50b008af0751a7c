"""FP8 expert weights for the first projection (W8A8) on the GPU against the oracle.

The gate / up weights are e4m3 with one fp32 scale per row (moe_quantize_rows_fp8, bit-exact to the
oracle's quantiser), each FFN input row is quantised the same way inside the call, and the tensor
cores run kind::f8f6f4 on the codes; h and the bf16 down projection follow.  Parity bar as for the
bf16 FFN: h and expert_out within the bar of the oracle's W8 FFN (expert_ffn_w8) on every row."""
import numpy as np
import pytest
import torch

import moe_inputs as mi
from _helpers import assert_close_bf16, bits16, bytes8, combine_magnitude, combine_row_atol, \
    ffn_row_atol, np_
from oracle import moe

pytestmark = pytest.mark.gpu


def quantize_gpu(x):
    import combine_moe_route_10_b200 as pkg
    rows, K = x.shape
    q = torch.empty((rows, K), dtype=torch.uint8, device="cuda")
    s = torch.empty(rows, dtype=torch.float32, device="cuda")
    pkg.moe_quantize_rows_fp8(x, rows, K, q, s)
    torch.cuda.synchronize()
    return q, s


def test_row_quantiser_is_bit_exact(cuda):
    g = torch.Generator(device="cuda").manual_seed(21)
    x = torch.randn(700, 1024, device="cuda", generator=g)
    x *= torch.exp(torch.empty(700, 1, device="cuda").uniform_(-60, 40, generator=g))
    x[3] = 0.0                                     # zero row: scale 1, codes 0
    x[4, :] = -0.0
    x[5, 7] = 1e-38                                # a row whose only value is tiny: subnormal scale
    x[5, :7] = 0.0
    x[5, 8:] = 0.0
    xb = x.to(torch.bfloat16)
    q, s = quantize_gpu(xb)
    q_ref, s_ref = moe.quantize_rows_fp8(xb.float().cpu().numpy())
    assert np.array_equal(np_(s).view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(bytes8(q), q_ref)


def w8_weights(d, E, F, H):
    gq, gs = quantize_gpu(d["w_gate"].view(E * F, H))
    uq, us = quantize_gpu(d["w_up"].view(E * F, H))
    # the GPU quantiser equals the oracle's: the oracle below uses the same codes and scales
    gq_ref, gs_ref = moe.quantize_rows_fp8(d["w_gate"].view(E * F, H).float().cpu().numpy())
    assert np.array_equal(bytes8(gq), gq_ref) and np.array_equal(np_(gs), gs_ref)
    return gq.view(E, F, H), gs.view(E, F), uq.view(E, F, H), us.view(E, F)


def check_w8(m, w, d, send, scales, off, S, gq, gs, uq, us, what):
    xin = moe.ffn_inputs(send, scales, w.payload == "fp8")
    h_ref, eo_ref = moe.expert_ffn_w8(xin, off, bytes8(gq).reshape(w.E, w.F, w.H), np_(gs),
                                      bytes8(uq).reshape(w.E, w.F, w.H), np_(us),
                                      bits16(d["w_down"]))
    assert_close_bf16(bits16(m.h_w8)[:S], h_ref, f"{what} h")
    assert_close_bf16(bits16(m.expert_out)[:S], eo_ref, f"{what} expert_out",
                      row_atol=ffn_row_atol(h_ref, off, d["w_down"]))
    return h_ref, eo_ref


@pytest.mark.parametrize("name", ["tiny", "train-small", "finegrained-small", "skewed-small"])
def test_w8_ffn_small_workloads(cuda, name):
    from combine_moe_route_10_b200 import MoeShuffle
    w = mi.get(name)
    d = mi.make_inputs(w, seed=4, device="cuda")
    cap = moe.capacity(w.capacity_factor, w.T, w.k, w.E)
    m = MoeShuffle(w.T, w.H, w.E, w.k, w.R, w.F, payload=w.payload, capacity=cap)
    gq, gs, uq, us = w8_weights(d, w.E, w.F, w.H)
    m.route(d["logits"])
    m.dispatch(d["x"])
    m.expert_ffn_w8(gq, gs, uq, us, d["w_down"])
    m.combine()
    assert m.status() == 0
    off = np_(m.expert_offsets)
    S = int(off[-1])
    send = bytes8(m.send)[:S] if w.payload == "fp8" else bits16(m.send)[:S]
    scales = np_(m.send_scales)[:S] if w.payload == "fp8" else None
    h_ref, eo_ref = check_w8(m, w, d, send, scales, off, S, gq, gs, uq, us, name)
    # the combine of the W8 expert outputs, every token
    sr, wt = np_(m.slot_row), np_(m.topk_w)
    y_ref = moe.combine(eo_ref, sr, wt, w.T, w.H)
    eo_atol = ffn_row_atol(h_ref, off, d["w_down"])
    assert_close_bf16(bits16(m.y), y_ref, f"{name} y", combine_magnitude(eo_ref, sr, wt),
                      combine_row_atol(eo_ref, sr, wt, eo_atol))
    # and the call is reproducible bit for bit
    eo1 = m.expert_out.clone()
    m.expert_ffn_w8(gq, gs, uq, us, d["w_down"])
    assert m.status() == 0
    assert torch.equal(m.expert_out[:S], eo1[:S])


@pytest.mark.parametrize("rows,H,F", [([40, 300, 0, 129], 320, 192),    # ragged H (half a k-step) and F
                                      ([1, 64, 65, 500], 256, 320)])
def test_w8_ffn_both_kernels_ragged(cuda, rows, H, F):
    from combine_moe_route_10_b200 import MoeShuffle
    E = len(rows)
    off = np.concatenate([[0], np.cumsum(rows)]).astype(np.int32)
    S = int(off[-1])
    g = torch.Generator(device="cuda").manual_seed(S + 7)
    x = mi.randn_bf16((S, H), g)
    d = {"w_gate": mi.randn_bf16((E, F, H), g, 0.05), "w_up": mi.randn_bf16((E, F, H), g, 0.05),
         "w_down": mi.randn_bf16((E, H, F), g, 0.05)}
    w = mi.Workload("w8-edge", S, H, E, 1, 1, F)
    m = MoeShuffle(S, H, E, 1, 1, F)
    gq, gs, uq, us = w8_weights(d, E, F, H)
    m.expert_ffn_w8(gq, gs, uq, us, d["w_down"], send=x, expert_offsets=torch.from_numpy(off).cuda())
    assert m.status() == 0
    check_w8(m, w, d, bits16(x), None, off, S, gq, gs, uq, us, str(rows))


def test_w8_ffn_full_size_skewed_every_row(cuda):
    """The default benchmark workload (skewed: T=16384, H=7168, E=128, top-2, capacity 320) with FP8
    gate / up weights, in the benchmark's launch configuration, on every packed row."""
    from combine_moe_route_10_b200 import MoeShuffle
    w = mi.get("skewed")
    d = mi.make_inputs(w, seed=0, device="cuda")
    cap = moe.capacity(w.capacity_factor, w.T, w.k, w.E)
    m = MoeShuffle(w.T, w.H, w.E, w.k, w.R, w.F, payload=w.payload, capacity=cap)
    gq, gs, uq, us = w8_weights(d, w.E, w.F, w.H)
    m.route(d["logits"])
    m.dispatch(d["x"])
    m.expert_ffn_w8(gq, gs, uq, us, d["w_down"])
    assert m.status() == 0
    off = np_(m.expert_offsets)
    S = int(off[-1])
    check_w8(m, w, d, bits16(m.send)[:S], None, off, S, gq, gs, uq, us, "skewed")
