"""GPU parity of the router, the dispatch and the combine against the CPU oracle, through the C ABI.

Bit-exact: expert ids, counts, offsets, slot rows, row tokens, permuted payload bytes and FP8
scales, and the combine output (both sides accumulate in fp32 in slot order with separately
rounded products and sums).  Routing weights: fp32 with expf on the GPU against fp64 in the
oracle, within rtol 4e-6 (expf <= 2 ulp, the fp32 subtraction of the maximum, k fp32 additions and
one division, each a few 2^-24)."""
import numpy as np
import pytest
import torch

import moe_inputs as mi
from _helpers import bits16, bytes8, np_
from oracle import moe

pytestmark = pytest.mark.gpu

ALL = list(mi.WORKLOADS)
W_RTOL, W_ATOL = 4e-6, 1e-7


def lib():
    import combine_moe_route_10_b200 as m
    m.load()
    return m


def gpu_route(logits: torch.Tensor, k: int, renorm: bool = True):
    m = lib()
    T, E = logits.shape
    idx = torch.full((T, k), -7, dtype=torch.int32, device=logits.device)
    w = torch.full((T, k), -7.0, dtype=torch.float32, device=logits.device)
    routed = torch.full((E,), -7, dtype=torch.int32, device=logits.device)
    m.moe_route(logits, T, E, k, renorm, idx, w, routed)
    torch.cuda.synchronize()
    return np_(idx), np_(w), np_(routed)


@pytest.mark.parametrize("renorm", [True, False])
@pytest.mark.parametrize("name", ALL)
def test_route_parity(cuda, name, renorm):
    w = mi.get(name)
    d = mi.make_inputs(w, seed=0, device="cuda", weights=False)
    idx, wt, routed = gpu_route(d["logits"], w.k, renorm)
    idx_ref, w_ref, routed_ref = moe.route(np_(d["logits"]), w.k, renorm)
    assert np.array_equal(idx, idx_ref)
    assert np.array_equal(routed, routed_ref)
    np.testing.assert_allclose(wt, w_ref, rtol=W_RTOL, atol=W_ATOL)


def test_route_ties_and_nonfinite(cuda):
    g = torch.Generator().manual_seed(5)
    ties = torch.randint(-3, 3, (500, 16), generator=g).float()       # many exact ties
    special = torch.tensor([[float("nan"), -float("inf"), 1.0, 1.0] + [-5.0] * 12,
                            [-float("inf")] * 16,
                            [0.0, float("inf"), 5.0, float("inf")] + [0.0] * 12,
                            [float("nan")] * 15 + [2.0],
                            [-0.0, 0.0] + [-1.0] * 14])
    sprinkled = torch.randn(300, 16, generator=g)
    mask = torch.rand(300, 16, generator=g)
    sprinkled[mask < 0.05] = float("nan")
    sprinkled[(mask >= 0.05) & (mask < 0.08)] = float("inf")
    sprinkled[(mask >= 0.08) & (mask < 0.12)] = -float("inf")
    for logits in (ties, special, sprinkled):
        for k in (1, 3, 16):
            for renorm in (True, False):
                idx, wt, routed = gpu_route(logits.cuda(), k, renorm)
                idx_ref, w_ref, routed_ref = moe.route(logits.numpy(), k, renorm)
                assert np.array_equal(idx, idx_ref)
                assert np.array_equal(routed, routed_ref)
                np.testing.assert_allclose(wt, w_ref, rtol=W_RTOL, atol=W_ATOL)


@pytest.mark.parametrize("T,E,k", [(1, 1, 1), (3, 5, 5), (64, 1024, 32), (200, 33, 7),
                                   (1000, 64, 1)])
def test_route_shapes(cuda, T, E, k):
    g = torch.Generator().manual_seed(T + E + k)
    logits = torch.randn(T, E, generator=g)
    idx, wt, routed = gpu_route(logits.cuda(), k)
    idx_ref, w_ref, routed_ref = moe.route(logits.numpy(), k)
    assert np.array_equal(idx, idx_ref) and np.array_equal(routed, routed_ref)
    np.testing.assert_allclose(wt, w_ref, rtol=W_RTOL, atol=W_ATOL)


def test_route_empty_clears_histogram(cuda):
    m = lib()
    routed = torch.full((8,), 5, dtype=torch.int32, device="cuda")
    dummy = torch.empty(0, device="cuda")
    m.moe_route(dummy, 0, 8, 2, True, dummy, dummy, routed)
    torch.cuda.synchronize()
    assert routed.sum().item() == 0


# ------------------------------------------------------------------------------------------------
def gpu_dispatch(x: torch.Tensor, idx_np: np.ndarray, E: int, R: int, cap: int, fp8: bool):
    from combine_moe_route_10_b200 import MoeShuffle
    T, H = x.shape
    k = idx_np.shape[1]
    m = MoeShuffle(T, H, E, k, R, 64, payload="fp8" if fp8 else "bf16", capacity=cap)
    m.dispatch(x, topk_idx=torch.from_numpy(np.ascontiguousarray(idx_np)).cuda())
    st = m.status()
    return m, st


def check_dispatch(m, plan, x_bits, fp8):
    S = plan["S"]
    assert np.array_equal(np_(m.expert_counts), plan["expert_counts"])
    assert np.array_equal(np_(m.expert_offsets), plan["expert_offsets"])
    assert np.array_equal(np_(m.rank_offsets), plan["rank_offsets"])
    assert np.array_equal(np_(m.slot_row), plan["slot_row"])
    assert np.array_equal(np_(m.row_token)[:S], plan["row_token"])
    send_ref, sc_ref = moe.dispatch_payload(x_bits, plan, fp8)
    if fp8:
        got = bytes8(m.send)[:S]
        assert np.array_equal(got, send_ref)
        assert np.array_equal(np_(m.send_scales)[:S].view(np.uint32), sc_ref.view(np.uint32))
    else:
        assert np.array_equal(bits16(m.send)[:S], send_ref)


@pytest.mark.parametrize("name", ALL)
def test_dispatch_parity(cuda, name):
    w = mi.get(name)
    d = mi.make_inputs(w, seed=0, device="cuda", weights=False)
    idx_ref, _, _ = moe.route(np_(d["logits"]), w.k)
    cap = moe.capacity(w.capacity_factor, w.T, w.k, w.E)
    plan = moe.dispatch_plan(idx_ref, w.E, w.R, cap)
    m, st = gpu_dispatch(d["x"], idx_ref, w.E, w.R, cap, w.payload == "fp8")
    assert st == 0
    check_dispatch(m, plan, bits16(d["x"]), w.payload == "fp8")


@pytest.mark.parametrize("case", ["one_expert", "cap1", "k_eq_E", "T1", "empty_experts",
                                  "ragged_T", "fp8_subnormal", "many_slots", "many_slots_fp8"])
def test_dispatch_edge_cases(cuda, case):
    g = np.random.default_rng(7)
    T, H, E, k, R, cap, fp8 = 300, 256, 8, 2, 4, 0, False
    if case == "one_expert":
        idx = np.stack([np.zeros(T), np.ones(T)], 1).astype(np.int32)  # every token: experts 0, 1
    elif case == "cap1":
        idx = np.argsort(-g.random((T, E)), 1)[:, :k].astype(np.int32)
        cap = 1
    elif case == "k_eq_E":
        k = E
        idx = np.argsort(-g.random((T, E)), 1).astype(np.int32)
        cap = 17
    elif case == "T1":
        T = 1
        idx = np.array([[5, 2]], dtype=np.int32)
    elif case == "empty_experts":
        E, R = 64, 8
        idx = np.argsort(-g.random((T, 4)), 1)[:, :k].astype(np.int32) * 16  # only 0,16,32,48
    elif case == "ragged_T":
        T, E, k, R, cap = 777, 128, 3, 16, 20
        idx = np.argsort(-(g.random((T, E)) + (np.arange(E) < 4) * 0.5), 1)[:, :k].astype(np.int32)
    elif case == "fp8_subnormal":
        fp8, H = True, 384
        idx = np.argsort(-g.random((T, E)), 1)[:, :k].astype(np.int32)
    elif case in ("many_slots", "many_slots_fp8"):
        # 1.9M slots, k = 32: thousands of rank/permute CTAs, each 256 slots spread over 64 experts
        T, E, k, R = 60000, 64, 32, 8
        fp8 = case == "many_slots_fp8"
        H, cap = (128, 25000) if fp8 else (64, 0)
        idx = np.argsort(-g.random((T, E)), 1)[:, :k].astype(np.int32)
    xf = g.normal(size=(T, H)).astype(np.float32)
    if case == "fp8_subnormal":
        xf[0, :128] = 0.0                      # all-zero block: scale 1, codes 0
        xf[1, 128:256] *= 1e-38                # tiny block: subnormal scale
        xf[2, :] = np.where(np.arange(H) % 2, -1e-7, 3.0)  # negative values that round to -0
    x_bits = (xf.view(np.uint32) >> 16).astype(np.uint16)
    x = torch.from_numpy(x_bits.view(np.int16)).view(torch.bfloat16).cuda()
    plan = moe.dispatch_plan(idx, E, R, cap)
    m, st = gpu_dispatch(x, idx, E, R, cap, fp8)
    assert st == 0
    check_dispatch(m, plan, x_bits, fp8)


def test_dispatch_invalid_expert_id_reports_status(cuda):
    m_ = lib()
    T, H, E, k = 64, 64, 8, 2
    idx = np.argsort(-np.random.default_rng(1).random((T, E)), 1)[:, :k].astype(np.int32)
    idx[10, 1] = E + 3
    idx[20, 0] = -1
    x = torch.randn(T, H).to(torch.bfloat16).cuda()
    m, st = gpu_dispatch(x, idx, E, 2, 0, False)
    assert st == m_.MOE_ERR_INVALID_TOPK
    sr = np_(m.slot_row)
    assert sr[10, 1] == -1 and sr[20, 0] == -1
    assert m.status() == 0                      # the status word was cleared by the read


def test_dispatch_is_deterministic(cuda):
    w = mi.get("skewed-small")
    d = mi.make_inputs(w, seed=3, device="cuda", weights=False)
    idx_ref, _, _ = moe.route(np_(d["logits"]), w.k)
    cap = moe.capacity(w.capacity_factor, w.T, w.k, w.E)
    m1, _ = gpu_dispatch(d["x"], idx_ref, w.E, w.R, cap, False)
    m2, _ = gpu_dispatch(d["x"], idx_ref, w.E, w.R, cap, False)
    S = int(m1.expert_offsets[w.E].item())
    assert S < w.T * w.k                         # this workload drops slots
    for a, b in [(m1.slot_row, m2.slot_row), (m1.row_token[:S], m2.row_token[:S]),
                 (m1.send[:S], m2.send[:S]), (m1.expert_offsets, m2.expert_offsets)]:
        assert torch.equal(a, b)


# ------------------------------------------------------------------------------------------------
@pytest.mark.parametrize("T,H,E,k,cap", [(100, 256, 8, 2, 0), (257, 1024, 16, 4, 30),
                                         (33, 7168, 256, 8, 2), (1, 64, 4, 4, 0),
                                         (2048, 512, 128, 2, 20)])
def test_combine_bit_exact(cuda, T, H, E, k, cap):
    m_ = lib()
    gen = torch.Generator().manual_seed(T * k + H)
    idx = mi.random_topk(T, E, k, gen).numpy()
    plan = moe.dispatch_plan(idx, E, 1, cap)
    S = plan["S"]
    eo = mi.randn_bf16((T * k, H), gen)
    wt = mi.random_weights_rows(T, k, gen)
    y_ref = moe.combine(bits16(eo)[:max(S, 1)], plan["slot_row"], wt.numpy(), T, H)
    y = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
    m_.moe_combine(eo.cuda(), T * k, torch.from_numpy(plan["slot_row"]).cuda(), wt.cuda(), T, k, H, y)
    torch.cuda.synchronize()
    assert np.array_equal(bits16(y), y_ref)


def test_combine_identity_experts_return_input(cuda):
    # expert_out = send (identity experts) with renormalised weights: y == x within one bf16 ulp
    from combine_moe_route_10_b200 import MoeShuffle
    for name in ["train", "skewed-small", "finegrained-small"]:
        w = mi.get(name)
        d = mi.make_inputs(w, seed=1, device="cuda", weights=False)
        m = MoeShuffle(w.T, w.H, w.E, w.k, w.R, 64, payload="bf16")   # no drop
        m.route(d["logits"])
        m.dispatch(d["x"])
        m.combine(expert_out=m.send)
        torch.cuda.synchronize()
        x = d["x"].float().cpu().numpy().astype(np.float64)
        y = m.y.float().cpu().numpy().astype(np.float64)
        ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(x), 1e-38))) - 7)
        assert np.all(np.abs(y - x) <= ulp)
        assert np.mean(y == x) > 0.95
