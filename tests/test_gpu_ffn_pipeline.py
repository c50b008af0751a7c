"""GPU parity of the grouped SwiGLU FFN and of the whole path against the CPU oracle (C ABI).

The FFN runs bf16 operands on the tensor cores with fp32 accumulation; the oracle accumulates in
fp64.  Both round h and the output to bf16.  Parity bar (per output tensor): max |gpu - ref| /
max |ref| <= 1e-2.  Small workloads are compared on every row; the full-size workloads on every
row too (train, skewed, finegrained FFN; decode's whole path), and on sampled rows (the first and
last row of sampled experts plus random rows), in the same launch configuration as the benchmark."""
import numpy as np
import pytest
import torch

import moe_inputs as mi
from _helpers import bits16, np_, rel_max_err, to_dev_bf16_from_bits
from oracle import moe

pytestmark = pytest.mark.gpu

RTOL = 1e-2
SMALL = ["tiny", "decode-small", "train-small", "finegrained-small", "skewed-small"]
FULL = ["decode", "train", "finegrained", "skewed"]


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
    assert rel_max_err(bits16(m.h)[:S], h_ref) <= RTOL
    assert rel_max_err(bits16(m.expert_out)[:S], y_ref) <= RTOL


def sample_rows(plan, n_experts, n_random, seed):
    off = plan["expert_offsets"]
    E = off.size - 1
    nonempty = [e for e in range(E) if off[e + 1] > off[e]]
    g = np.random.default_rng(seed)
    big = sorted(nonempty, key=lambda e: off[e] - off[e + 1])[:2]      # the largest experts
    pick = set(big) | set(g.choice(nonempty, size=min(n_experts, len(nonempty)), replace=False))
    rows = {}
    for e in sorted(pick):
        lo, hi = int(off[e]), int(off[e + 1])
        r = {lo, hi - 1} | set(g.integers(lo, hi, size=n_random).tolist())
        rows[e] = np.array(sorted(r))
    return rows


def oracle_rows(w, d, xin, rows_by_expert):
    """Oracle FFN output for selected rows, expert by expert (weights copied per expert)."""
    out = {}
    for e, r in rows_by_expert.items():
        wg, wu, wd = (bits16(d[n][e:e + 1]) for n in ("w_gate", "w_up", "w_down"))
        h, y = moe.expert_ffn(xin[r], np.array([0, r.size]), wg, wu, wd)
        out[e] = (h, y)
    return out


@pytest.mark.parametrize("name", FULL)
def test_ffn_parity_full_size_sampled(cuda, name):
    w = mi.get(name)
    d = mi.make_inputs(w, seed=0, device="cuda")
    _, _, plan, send, scales = oracle_plan(w, d)
    m, _ = shuffle_for(w)
    run_gpu_ffn_on_oracle_rows(m, w, plan, send, scales, d)
    rows = sample_rows(plan, n_experts=4, n_random=6, seed=1)
    all_rows = np.concatenate(list(rows.values()))
    xin = moe.ffn_inputs(send[all_rows], None if scales is None else scales[all_rows],
                         w.payload == "fp8")
    xin_full = np.zeros((plan["S"], w.H))
    xin_full[all_rows] = xin
    ref = oracle_rows(w, d, xin_full, rows)
    h_gpu, y_gpu = bits16(m.h), bits16(m.expert_out)
    for e, r in rows.items():
        h_ref, y_ref = ref[e]
        assert rel_max_err(h_gpu[r], h_ref) <= RTOL, e
        assert rel_max_err(y_gpu[r], y_ref) <= RTOL, e


@pytest.mark.parametrize("name", ["train", "skewed", "finegrained"])
def test_ffn_parity_full_size_all_rows(cuda, name):
    """Full size, every packed row, in the benchmark's launch configuration: train (tensor-bound;
    experts of 300-2300 rows: full 128-row blocks and ragged last blocks), skewed (capacity-capped
    experts of 2-3 blocks) and finegrained (FP8 payload; 256 experts from 1 row to 32 blocks).
    The oracle runs expert by expert with that expert's weights only."""
    w = mi.get(name)
    d = mi.make_inputs(w, seed=0, device="cuda")
    _, _, plan, send, scales = oracle_plan(w, d)
    m, _ = shuffle_for(w)
    run_gpu_ffn_on_oracle_rows(m, w, plan, send, scales, d)
    xin = moe.ffn_inputs(send, scales, w.payload == "fp8")
    off = plan["expert_offsets"]
    rows = {e: np.arange(off[e], off[e + 1]) for e in range(w.E) if off[e + 1] > off[e]}
    ref = oracle_rows(w, d, xin, rows)
    S = plan["S"]
    h_ref = np.concatenate([ref[e][0] for e in sorted(ref)])
    y_ref = np.concatenate([ref[e][1] for e in sorted(ref)])
    assert h_ref.shape[0] == S
    assert rel_max_err(bits16(m.h)[:S], h_ref) <= RTOL
    assert rel_max_err(bits16(m.expert_out)[:S], y_ref) <= RTOL


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
    assert rel_max_err(bits16(m.expert_out)[:o["S"]], o["expert_out"]) <= RTOL
    assert rel_max_err(bits16(y), o["y"]) <= RTOL


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
    assert rel_max_err(bits16(m.h)[:o["S"]], o["h"]) <= RTOL
    assert rel_max_err(bits16(m.expert_out)[:o["S"]], o["expert_out"]) <= RTOL
    assert rel_max_err(bits16(y), o["y"]) <= RTOL
    # the combine is exact given its inputs: the oracle's combine of the GPU's expert outputs
    assert np.array_equal(bits16(y), moe.combine(bits16(m.expert_out), np_(m.slot_row),
                                                 np_(m.topk_w), w.T, w.H))


@pytest.mark.parametrize("name", FULL)
def test_pipeline_full_size_sampled_tokens(cuda, name):
    """The benchmark's launch configuration at full size; oracle on a token sample."""
    w = mi.get(name)
    d = mi.make_inputs(w, seed=0, device="cuda")
    m, cap = shuffle_for(w)
    y = m.forward(d["logits"], d["x"], d["w_gate"], d["w_up"], d["w_down"])
    assert m.status() == 0
    idx, wt, plan, send, scales = oracle_plan(w, d)
    assert np.array_equal(np_(m.slot_row), plan["slot_row"])
    g = np.random.default_rng(4)
    toks = np.unique(np.concatenate([[0, w.T - 1], g.integers(0, w.T, size=6)]))
    sr = plan["slot_row"][toks]
    rows = sr[sr >= 0]
    by_e = {}
    off = plan["expert_offsets"]
    for r in rows:
        e = int(np.searchsorted(off, r, side="right") - 1)
        by_e.setdefault(e, []).append(int(r))
    by_e = {e: np.array(sorted(v)) for e, v in by_e.items()}
    xin_full = np.zeros((plan["S"], w.H))
    xin_full[rows] = moe.ffn_inputs(send[rows], None if scales is None else scales[rows],
                                    w.payload == "fp8")
    ref = oracle_rows(w, d, xin_full, by_e)
    y_e = np.full((plan["S"], w.H), 0x7FC0, dtype=np.uint16)
    for e, r in by_e.items():
        y_e[r] = ref[e][1]
    y_ref = moe.combine(y_e, sr, wt[toks], toks.size, w.H)
    assert rel_max_err(bits16(y)[toks], y_ref) <= RTOL


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
        assert rel_max_err(bits16(m.expert_out)[:o["S"]], o["expert_out"]) <= RTOL
        assert rel_max_err(bits16(y), o["y"]) <= RTOL


@pytest.mark.parametrize("rows", [
    [150, 200, 256, 129, 180, 222, 140, 255],          # every expert: two 128-row blocks
    [150, 200, 256, 40, 300, 129, 0, 180],             # mostly two blocks, plus 1-, 3- and 0-block
    [130, 0, 0, 0, 0, 0, 0, 0],                        # a single two-block expert
])
def test_ffn_two_block_experts(cuda, rows):
    """Experts with 129..256 rows run as 256-row tiles (two MMAs sharing one weight tile) when
    they are the majority; other experts keep 128-row tiles in the same launch."""
    from combine_moe_route_10_b200 import MoeShuffle
    E, H, F = len(rows), 256, 320
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
    assert rel_max_err(bits16(m.h)[:S], h_ref) <= RTOL
    assert rel_max_err(bits16(m.expert_out)[:S], y_ref) <= RTOL


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
    if o["S"]:
        assert rel_max_err(bits16(m.expert_out)[:o["S"]], o["expert_out"]) <= RTOL
    assert rel_max_err(bits16(y), o["y"]) <= RTOL
