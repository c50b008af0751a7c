"""GPU parity of the grouped SwiGLU FFN and of the whole path against the CPU oracle (C ABI).

The FFN runs bf16 operands on the tensor cores with fp32 accumulation; the oracle accumulates in
fp64.  Both round h and the output to bf16.  Parity bar per bf16 output tensor: max |gpu - ref| /
max |ref| <= 1e-2, and no element outside 1e-2 |ref| + 1e-3 max |ref|, plus for expert_out the
row allowance of four one-ulp flips of h, and for y the expert_out allowance carried through the
combine weights with the size of the summands as magnitude (assert_ffn_and_combine).
Every workload is compared on every packed row and every token: the small ones through the whole
path, the full-size ones in the benchmark's launch configuration."""
import numpy as np
import pytest
import torch

import moe_inputs as mi
from _helpers import assert_ffn_and_combine, bits16, np_, to_dev_bf16_from_bits
from oracle import moe

pytestmark = pytest.mark.gpu

SMALL = ["tiny", "decode-small", "train-small", "finegrained-small", "skewed-small"]


def shuffle_for(w):
    from combine_moe_route_10_b200 import MoeShuffle
    cap = moe.capacity(w.capacity_factor, w.T, w.k, w.E)
    return MoeShuffle(w.T, w.H, w.E, w.k, w.R, w.F, payload=w.payload, capacity=cap), cap


def oracle_plan(w, d):
    idx, wt, _ = moe.route(np_(d["logits"]), w.k)
    cap = moe.capacity(w.capacity_factor, w.T, w.k, w.E)
    plan = moe.dispatch_plan(idx, w.E, w.R, cap)
    send, scales = moe.dispatch_payload(bits16(d["x"]), plan, w.payload == "fp8")
    return idx, wt, plan, send, scales


def run_gpu_ffn_on_oracle_rows(m, w, plan, send, scales, d):
    """GPU FFN with the oracle's packed rows and offsets as inputs."""
    S = plan["S"]
    if w.payload == "fp8":
        send_dev = torch.zeros((m.max_rows, w.H), dtype=torch.uint8, device="cuda")
        send_dev[:S] = torch.from_numpy(send).cuda()
        sc_dev = torch.zeros((m.max_rows, w.H // 128), dtype=torch.float32, device="cuda")
        sc_dev[:S] = torch.from_numpy(scales).cuda()
    else:
        send_dev = torch.zeros((m.max_rows, w.H), dtype=torch.bfloat16, device="cuda")
        send_dev[:S] = to_dev_bf16_from_bits(send, "cuda")
        sc_dev = None
    off = torch.from_numpy(plan["expert_offsets"]).cuda()
    m.expert_ffn(d["w_gate"], d["w_up"], d["w_down"], send=send_dev, send_scales=sc_dev,
                 expert_offsets=off)
    assert m.status() == 0


@pytest.mark.parametrize("name", SMALL)
def test_ffn_parity_all_rows(cuda, name):
    w = mi.get(name)
    d = mi.make_inputs(w, seed=0, device="cuda")
    _, _, plan, send, scales = oracle_plan(w, d)
    m, _ = shuffle_for(w)
    run_gpu_ffn_on_oracle_rows(m, w, plan, send, scales, d)
    xin = moe.ffn_inputs(send, scales, w.payload == "fp8")
    h_ref, y_ref = moe.expert_ffn(xin, plan["expert_offsets"], bits16(d["w_gate"]),
                                  bits16(d["w_up"]), bits16(d["w_down"]))
    S = plan["S"]
    assert_ffn_and_combine(bits16(m.h)[:S], bits16(m.expert_out)[:S], None, h_ref, y_ref, None,
                           plan["expert_offsets"], d["w_down"], None, None, name)


def oracle_rows(w, d, xin, rows_by_expert):
    """Oracle FFN output for selected rows, expert by expert (weights copied per expert)."""
    out = {}
    for e, r in rows_by_expert.items():
        wg, wu, wd = (bits16(d[n][e:e + 1]) for n in ("w_gate", "w_up", "w_down"))
        h, y = moe.expert_ffn(xin[r], np.array([0, r.size]), wg, wu, wd)
        out[e] = (h, y)
    return out


@pytest.mark.parametrize("name", ["train", "skewed", "finegrained"])
def test_pipeline_full_size_every_row_and_token(cuda, name):
    """Full size, in the benchmark's launch configuration, nothing sampled: train (tensor-bound;
    experts of 300-2300 rows: full 128-row blocks and ragged last blocks), skewed (capacity-capped
    experts of 2-3 blocks, 12k dropped slots) and finegrained (FP8 payload; 256 experts from 0 rows
    to 32 blocks).  Routing, plan and payload bit-exact; h and expert_out on every packed row and y
    on every token within the parity bar; y also bit-exact against the oracle's combine of the
    GPU's own expert outputs.  The oracle FFN runs expert by expert with that expert's weights."""
    w = mi.get(name)
    fp8 = w.payload == "fp8"
    d = mi.make_inputs(w, seed=0, device="cuda")
    m, _ = shuffle_for(w)
    y = m.forward(d["logits"], d["x"], d["w_gate"], d["w_up"], d["w_down"])
    assert m.status() == 0
    idx, wt, plan, send, scales = oracle_plan(w, d)
    S = plan["S"]
    assert np.array_equal(np_(m.topk_idx), idx)
    np.testing.assert_allclose(np_(m.topk_w), wt, rtol=4e-6, atol=1e-7)
    for key in ("expert_counts", "expert_offsets", "rank_offsets", "slot_row"):
        assert np.array_equal(np_(getattr(m, key)), plan[key]), key
    assert np.array_equal(np_(m.row_token)[:S], plan["row_token"])
    if fp8:
        assert np.array_equal(np_(m.send.view(torch.uint8))[:S], send)
        assert np.array_equal(np_(m.send_scales)[:S].view(np.uint32), scales.view(np.uint32))
    else:
        assert np.array_equal(bits16(m.send)[:S], send)
    xin = moe.ffn_inputs(send, scales, fp8)
    off = plan["expert_offsets"]
    rows = {e: np.arange(off[e], off[e + 1]) for e in range(w.E) if off[e + 1] > off[e]}
    ref = oracle_rows(w, d, xin, rows)
    h_ref = np.concatenate([ref[e][0] for e in sorted(ref)])
    y_ref = np.concatenate([ref[e][1] for e in sorted(ref)])
    del ref, xin
    assert h_ref.shape[0] == S
    eo = bits16(m.expert_out)[:S]
    y_bits = bits16(y)
    # the combine is exact given its inputs: every token
    assert np.array_equal(y_bits, moe.combine(eo, np_(m.slot_row), np_(m.topk_w), w.T, w.H))
    # h and expert_out on every packed row, y on every token, against the oracle's expert outputs
    # and routing weights
    assert_ffn_and_combine(bits16(m.h)[:S], eo, y_bits, h_ref, y_ref,
                           moe.combine(y_ref, plan["slot_row"], wt, w.T, w.H), off, d["w_down"],
                           plan["slot_row"], wt, name)


@pytest.mark.parametrize("name", ["finegrained", "skewed"])
def test_ffn_bit_reproducible_under_run_time_scheduling(cuda, name):
    """Tiles are claimed at run time, so consecutive calls schedule them differently; every output
    element still comes from one tile with a fixed k order, so the results are bit-identical."""
    w = mi.get(name)
    d = mi.make_inputs(w, seed=0, device="cuda")
    m, _ = shuffle_for(w)
    m.route(d["logits"])
    m.dispatch(d["x"])
    outs = []
    for _ in range(3):
        m.expert_ffn(d["w_gate"], d["w_up"], d["w_down"])
        outs.append((m.h.clone(), m.expert_out.clone()))
    assert m.status() == 0
    S = int(m.expert_offsets[w.E].item())
    for h, y in outs[1:]:
        assert torch.equal(h[:S], outs[0][0][:S])
        assert torch.equal(y[:S], outs[0][1][:S])


@pytest.mark.parametrize("name", SMALL)
def test_pipeline_end_to_end(cuda, name):
    w = mi.get(name)
    d = mi.make_inputs(w, seed=2, device="cuda")
    m, cap = shuffle_for(w)
    y = m.forward(d["logits"], d["x"], d["w_gate"], d["w_up"], d["w_down"])
    assert m.status() == 0
    o = moe.pipeline(np_(d["logits"]), bits16(d["x"]), bits16(d["w_gate"]), bits16(d["w_up"]),
                     bits16(d["w_down"]), w.k, w.R, w.capacity_factor, w.payload == "fp8")
    assert np.array_equal(np_(m.topk_idx), o["topk_idx"])
    assert np.array_equal(np_(m.slot_row), o["slot_row"])
    assert np.array_equal(np_(m.expert_offsets), o["expert_offsets"])
    assert_ffn_and_combine(bits16(m.h)[:o["S"]], bits16(m.expert_out)[:o["S"]], bits16(y), o["h"],
                           o["expert_out"], o["y"], o["expert_offsets"], d["w_down"],
                           o["slot_row"], o["topk_w"], name)


def test_pipeline_decode_full_size_every_token(cuda):
    """The benchmark's default workload at full size (T=128, H=4096, E=8, F=14336, the bench's seed)
    in the bench's launch configuration: every token and every packed row against the oracle."""
    w = mi.get("decode")
    d = mi.make_inputs(w, seed=0, device="cuda")
    m, _ = shuffle_for(w)
    y = m.forward(d["logits"], d["x"], d["w_gate"], d["w_up"], d["w_down"])
    assert m.status() == 0
    o = moe.pipeline(np_(d["logits"]), bits16(d["x"]), bits16(d["w_gate"]), bits16(d["w_up"]),
                     bits16(d["w_down"]), w.k, w.R, w.capacity_factor, w.payload == "fp8")
    assert np.array_equal(np_(m.topk_idx), o["topk_idx"])
    assert np.array_equal(np_(m.slot_row), o["slot_row"])
    assert np.array_equal(np_(m.expert_offsets), o["expert_offsets"])
    assert np.array_equal(bits16(m.send)[:o["S"]], o["send"])
    assert_ffn_and_combine(bits16(m.h)[:o["S"]], bits16(m.expert_out)[:o["S"]], bits16(y), o["h"],
                           o["expert_out"], o["y"], o["expert_offsets"], d["w_down"],
                           o["slot_row"], o["topk_w"], "decode")
    # the combine is exact given its inputs: the oracle's combine of the GPU's expert outputs
    assert np.array_equal(bits16(y), moe.combine(bits16(m.expert_out), np_(m.slot_row),
                                                 np_(m.topk_w), w.T, w.H))


def test_ffn_workspace_reused_across_calls_with_different_routing(cuda):
    """One FFN workspace, consecutive calls whose expert offsets differ: the GEMM-1 completion
    counters inside the workspace return to zero after every call."""
    w = mi.get("train-small")
    m, _ = shuffle_for(w)
    for seed in (0, 1, 2):
        d = mi.make_inputs(w, seed=seed, device="cuda")
        y = m.forward(d["logits"], d["x"], d["w_gate"], d["w_up"], d["w_down"])
        assert m.status() == 0
        o = moe.pipeline(np_(d["logits"]), bits16(d["x"]), bits16(d["w_gate"]), bits16(d["w_up"]),
                         bits16(d["w_down"]), w.k, w.R)
        assert np.array_equal(np_(m.expert_offsets), o["expert_offsets"])
        assert_ffn_and_combine(bits16(m.h)[:o["S"]], bits16(m.expert_out)[:o["S"]], bits16(y),
                               o["h"], o["expert_out"], o["y"], o["expert_offsets"], d["w_down"],
                               o["slot_row"], o["topk_w"], f"seed {seed}")


@pytest.mark.parametrize("rows,H,F", [
    ([150, 200, 256, 129, 180, 222, 140, 255], 256, 320),  # every expert: two 128-row blocks
    ([150, 200, 256, 40, 300, 129, 0, 180], 256, 320),     # plus 1-, 3- and 0-block experts
    ([130, 0, 0, 0, 0, 0, 0, 0], 256, 320),                # a single two-block expert
    # the kernel limits: 64 rows (single CTA) / 65 (a pair whose second block is empty); 256 / 257
    # and 512 / 513 (one, two and three pairs); ragged H (the second 256-column block half out)
    ([64, 65, 80, 96, 256, 257, 511, 512, 513, 17], 320, 192),
    ([65, 512, 513, 1000], 64, 128),                       # one k-step of GEMM-1, F below 128 cols
])
def test_ffn_two_block_experts(cuda, rows, H, F):
    """Experts of 65..256 rows (two 128-row blocks, the second one ragged or empty) next to experts
    of one, three, four and more blocks and empty ones: each pair of blocks is one 2-CTA tile, and
    the blocks of an expert read the same weight column blocks."""
    from combine_moe_route_10_b200 import MoeShuffle
    E = len(rows)
    off = np.concatenate([[0], np.cumsum(rows)]).astype(np.int32)
    S = int(off[-1])
    g = torch.Generator(device="cuda").manual_seed(sum(rows))
    x = mi.randn_bf16((S, H), g)
    wg, wu = mi.randn_bf16((E, F, H), g, 0.05), mi.randn_bf16((E, F, H), g, 0.05)
    wd = mi.randn_bf16((E, H, F), g, 0.05)
    m = MoeShuffle(S, H, E, 1, 1, F)                   # max_rows = S
    m.expert_ffn(wg, wu, wd, send=x, expert_offsets=torch.from_numpy(off).cuda())
    assert m.status() == 0
    h_ref, y_ref = moe.expert_ffn(moe.ffn_inputs(bits16(x), None, False), off, bits16(wg),
                                  bits16(wu), bits16(wd))
    assert_ffn_and_combine(bits16(m.h)[:S], bits16(m.expert_out)[:S], None, h_ref, y_ref, None, off,
                           wd, None, None, str(rows))


@pytest.mark.parametrize("T,H,E,k,R,F,payload,cf", [
    (0, 128, 4, 2, 2, 128, "bf16", 0.0),      # empty batch
    (1, 128, 1, 1, 1, 128, "bf16", 0.0),      # one token, one expert: a dense SwiGLU MLP
    (3, 64, 2, 2, 1, 64, "bf16", 0.0),        # 6 rows in all, one k-block, F below the tile
    (5, 256, 4, 1, 2, 192, "fp8", 0.0),       # FP8 payload, tiny T
    (64, 320, 16, 4, 4, 64, "bf16", 1.0),     # H not a multiple of 256, drops at capacity 16
    (200, 192, 8, 8, 8, 128, "bf16", 0.0),    # k = E
    (64, 128, 1024, 32, 32, 64, "bf16", 0.0),  # E and k at their limits: ~2 rows per expert
    (64, 128, 1024, 32, 32, 64, "fp8", 1.0),   # the same with the FP8 payload and capacity 2
])
def test_pipeline_edge_shapes(cuda, T, H, E, k, R, F, payload, cf):
    from combine_moe_route_10_b200 import MoeShuffle
    w = mi.Workload("edge", T, H, E, k, R, F, payload=payload, capacity_factor=cf)
    d = mi.make_inputs(w, seed=9, device="cuda")
    cap = moe.capacity(cf, T, k, E)
    m = MoeShuffle(T, H, E, k, R, F, payload=payload, capacity=cap)
    y = m.forward(d["logits"], d["x"], d["w_gate"], d["w_up"], d["w_down"])
    assert m.status() == 0
    o = moe.pipeline(np_(d["logits"]), bits16(d["x"]), bits16(d["w_gate"]), bits16(d["w_up"]),
                     bits16(d["w_down"]), k, R, cf, payload == "fp8")
    assert np.array_equal(np_(m.expert_offsets), o["expert_offsets"])
    assert np.array_equal(np_(m.slot_row), o["slot_row"])
    if T == 0:
        assert y.numel() == 0
        return
    assert_ffn_and_combine(bits16(m.h)[:o["S"]], bits16(m.expert_out)[:o["S"]], bits16(y), o["h"],
                           o["expert_out"], o["y"], o["expert_offsets"], d["w_down"],
                           o["slot_row"], o["topk_w"], "edge")
