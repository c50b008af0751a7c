"""Failure detection on the GPU without a fault: a bounded device wait is made to run out.

The fused FFN's GEMM-2 tiles wait (bounded, about one second) on per-row-block completion counters
in the workspace.  Setting those counters to a value that the GEMM-1 epilogues can never raise to
the target is a flag that nothing sets: the waits run out, the kernel records MOE_ERR_TIMEOUT in the
workspace status word, drains its own copies and MMAs, frees TMEM and returns.  The context stays
usable: after re-zeroing the workspace the same call gives correct results again."""
import pytest
import torch

import moe_inputs as mi
from _helpers import assert_ffn_and_combine, bits16, np_
from oracle import moe

pytestmark = pytest.mark.gpu


def counter_slice(m, w):
    """int32 view of the GEMM-1 completion counters inside the FFN workspace."""
    def r256(b):
        return (b + 255) // 256 * 256
    off = 256 + r256(m.max_rows * w.F * 2)
    if w.payload == "fp8":
        off += r256(m.max_rows * w.H * 2)
    n = m.max_rows // 128 + w.E + 1
    return m.ws_ffn[off:off + 4 * n].view(torch.int32)


def test_ffn_wait_timeout_is_reported_and_recoverable(cuda):
    import combine_moe_route_10_b200 as pkg
    from combine_moe_route_10_b200 import MoeShuffle
    w = mi.get("train-small")
    d = mi.make_inputs(w, seed=5, device="cuda")
    m = MoeShuffle(w.T, w.H, w.E, w.k, w.R, w.F)
    m.forward(d["logits"], d["x"], d["w_gate"], d["w_up"], d["w_down"])
    assert m.status() == pkg.MOE_OK
    y_ok = m.y.clone()

    counter_slice(m, w).fill_(-(1 << 30))          # no GEMM-1 epilogue can reach the target now
    torch.cuda.synchronize()
    m.expert_ffn(d["w_gate"], d["w_up"], d["w_down"])
    st = pkg.moe_sync_status(m.ws_ffn)
    assert st == pkg.MOE_ERR_TIMEOUT
    assert torch.cuda.is_available() and torch.ones(4, device="cuda").sum().item() == 4.0

    m.ws_ffn.zero_()                               # documented recovery: zero-fill the workspace
    m.forward(d["logits"], d["x"], d["w_gate"], d["w_up"], d["w_down"])
    assert m.status() == pkg.MOE_OK
    assert torch.equal(m.y, y_ok)
    o = moe.pipeline(np_(d["logits"]), bits16(d["x"]), bits16(d["w_gate"]), bits16(d["w_up"]),
                     bits16(d["w_down"]), w.k, w.R)
    assert_ffn_and_combine(bits16(m.h)[:o["S"]], bits16(m.expert_out)[:o["S"]], bits16(m.y), o["h"],
                           o["expert_out"], o["y"], o["expert_offsets"], d["w_down"],
                           o["slot_row"], o["topk_w"], "after recovery")


@pytest.mark.parametrize("bad", [[0, 90, 150, 400], [-50, 90, 150, 200]])
def test_expert_offsets_outside_the_buffers_are_clamped(cuda, bad):
    """Expert offsets past max_rows or below zero (a caller's mistake, not a fault): the FFN and the
    expert backward clamp them to [0, max_rows], so every result equals the one for the clamped
    offsets, and the rows past max_rows in oversized output buffers keep their contents."""
    from combine_moe_route_10_b200 import _lib
    E, H, F, S, SPARE = 3, 128, 128, 200, 64
    g = torch.Generator(device="cuda").manual_seed(5)
    x = mi.randn_bf16((S, H), g)
    d_eo = mi.randn_bf16((S, H), g)
    wg, wu = mi.randn_bf16((E, F, H), g, 0.05), mi.randn_bf16((E, F, H), g, 0.05)
    wd = mi.randn_bf16((E, H, F), g, 0.05)
    good = torch.tensor([0, 90, 150, 200], dtype=torch.int32, device="cuda")
    sentinel = torch.full((SPARE, H), 7.0, dtype=torch.bfloat16, device="cuda")

    def forward(off):
        eo = torch.zeros((S + SPARE, H), dtype=torch.bfloat16, device="cuda")
        eo[S:] = sentinel
        nb = _lib.moe_ffn_workspace_size(S, E, H, F, _lib.MOE_PAYLOAD_BF16)
        ws = torch.zeros(nb, dtype=torch.uint8, device="cuda")
        _lib.moe_expert_ffn(x, None, _lib.MOE_PAYLOAD_BF16, off, S, E, H, F, wg, wu, wd, eo, ws, nb)
        assert _lib.moe_sync_status(ws) == _lib.MOE_OK
        return eo

    def backward(off):
        dx_rows = torch.zeros((S + SPARE, H), dtype=torch.bfloat16, device="cuda")
        dx_rows[S:] = sentinel
        grads = [torch.zeros((E, F, H), dtype=torch.float32, device="cuda") for _ in range(2)]
        dwd = torch.zeros((E, H, F), dtype=torch.float32, device="cuda")
        nb = _lib.moe_expert_backward_workspace_size(S, F)
        ws = torch.zeros(nb, dtype=torch.uint8, device="cuda")
        _lib.moe_expert_backward(x, d_eo, off, S, E, H, F, wg, wu, wd, dx_rows, grads[0], grads[1],
                                 dwd, ws, nb)
        assert _lib.moe_sync_status(ws) == _lib.MOE_OK
        return dx_rows, grads[0], grads[1], dwd

    off_bad = torch.tensor(bad, dtype=torch.int32, device="cuda")
    eo_bad, eo_good = forward(off_bad), forward(good)
    assert torch.equal(eo_bad, eo_good)
    assert torch.equal(eo_bad[S:], sentinel)
    for a, b in zip(backward(off_bad), backward(good)):
        assert torch.equal(a, b)
    assert torch.equal(backward(off_bad)[0][S:], sentinel)
