"""Expert parallelism on the GPU through the C ABI.

* ``moe_ep_regroup`` against the oracle's segment layouts, bit for bit: both orders on both sides,
  packed and padded blocks, 16-byte and 4-byte rows, the second payload, the expert offsets, rows
  outside the segments left untouched; counts that do not fit (negative, longer than a block's
  stride, more than a buffer holds) copy nothing and report MOE_ERR_INVALID_COUNTS.
* ``MoeEP`` over R = 4 ranks emulated by threads on one GPU (the all-to-all is a copy between the
  ranks' buffers, no kernel waits on another) must give every rank exactly its slice of the
  single-device path over all ranks' tokens, in both exchange modes and both payloads; one small
  case is also held to the oracle's parity bar.
* ``moe_ep_exchange`` (the exchange over peer memory fused with the regrouping) against the
  oracle-backed restatement, pulling from and pushing into separate buffers of every rank; counts
  that do not fit copy nothing and report MOE_ERR_INVALID_COUNTS.
* ``MoeEP`` over a real NCCL process group of one rank, eager and captured in a CUDA graph (the
  low-latency and peer-memory modes need no host synchronisation), and through torch symmetric
  memory.
"""
import socket

import numpy as np
import pytest
import torch

import moe_inputs as mi
from _ep_loopback import run_ranks
from _helpers import assert_ffn_and_combine, bits16, bytes8, np_
from oracle import moe

pytestmark = pytest.mark.gpu


def _regroup(counts, A, B, so, ss, src, do, ds, dst, src_aux=None, dst_aux=None, offs=None,
             status=None):
    from combine_moe_route_10_b200 import _lib
    _lib.moe_ep_regroup(counts, A, B, so, ss, src.shape[0], do, ds, dst.shape[0], src, dst,
                        src[0].numel() * src.element_size(), src_aux, dst_aux,
                        0 if src_aux is None else src_aux[0].numel() * src_aux.element_size(),
                        offs, status)


@pytest.mark.parametrize("so,do", [(0, 1), (1, 0), (0, 0), (1, 1)])
@pytest.mark.parametrize("padded_src,padded_dst", [(False, False), (True, False), (False, True)])
@pytest.mark.parametrize("width", [256, 7])           # bf16 [.., 256]: 512-byte rows; 7 fp32 words
def test_regroup_matches_oracle(cuda, so, do, padded_src, padded_dst, width):
    from combine_moe_route_10_b200 import _lib
    g = np.random.default_rng(so * 7 + do + width)
    A, B = 5, 6
    counts = g.integers(0, 40, size=(A, B)).astype(np.int32)
    counts[2, :] = 0
    counts[:, 4] = 0
    n = int(counts.sum())
    blk_s = counts.sum(axis=1 if so == 0 else 0)
    blk_d = counts.sum(axis=1 if do == 0 else 0)
    ss = int(blk_s.max()) + 3 if padded_src else 0
    ds = int(blk_d.max()) + 5 if padded_dst else 0
    rows_s = (A if so == 0 else B) * ss if ss else n
    rows_d = (A if do == 0 else B) * ds if ds else n
    if width == 256:
        src = torch.randn(rows_s, width, device=cuda).to(torch.bfloat16)
        dst = torch.full((rows_d + 3, width), 7.0, device=cuda, dtype=torch.bfloat16)
    else:
        src = torch.randn(rows_s, width, device=cuda)
        dst = torch.full((rows_d + 3, width), 7.0, device=cuda)
    aux_s = torch.randn(rows_s, 3, device=cuda)
    aux_d = torch.full((rows_d + 3, 3), -1.0, device=cuda)
    offs = torch.full((B + 1,), -9, dtype=torch.int32, device=cuda)
    status = torch.zeros(64, dtype=torch.int32, device=cuda)
    c = torch.from_numpy(counts).to(cuda)
    dst0 = bytes8(dst).reshape(rows_d + 3, -1).copy()     # rows outside the segments stay as is
    aux0 = np_(aux_d).copy()
    _regroup(c, A, B, so, ss, src, do, ds, dst, aux_s, aux_d, offs, status)
    assert _lib.moe_sync_status(status) == 0
    exp, off = moe.ep_regroup(counts, bytes8(src).reshape(rows_s, -1), so, ss, dst0, do, ds)
    assert np.array_equal(bytes8(dst).reshape(rows_d + 3, -1), exp)
    exp_aux, _ = moe.ep_regroup(counts, np_(aux_s), so, ss, aux0, do, ds)
    assert np.array_equal(np_(aux_d), exp_aux)
    assert np.array_equal(np_(offs), off)


def test_regroup_rejects_counts_that_do_not_fit(cuda):
    from combine_moe_route_10_b200 import _lib
    A, B, M = 3, 2, 10
    src = torch.randn(A * M, 64, device=cuda).to(torch.bfloat16)
    status = torch.zeros(64, dtype=torch.int32, device=cuda)
    cases = [
        np.array([[1, 2], [-1, 3], [0, 0]]),           # a negative count
        np.array([[6, 5], [0, 0], [1, 1]]),            # block 0 holds 11 rows > stride 10
        np.array([[9, 0], [9, 0], [9, 9]]),            # 36 rows > the 30-row destination
    ]
    for counts in cases:
        dst = torch.zeros(A * M, 64, device=cuda, dtype=torch.bfloat16)
        _regroup(torch.from_numpy(counts.astype(np.int32)).to(cuda), A, B, 0, M, src, 1, 0, dst,
                 status=status)
        assert _lib.moe_sync_status(status) == _lib.MOE_ERR_INVALID_COUNTS, counts
        assert int(dst.abs().sum().item()) == 0
    # and a fitting one still works afterwards
    dst = torch.zeros(A * M, 64, device=cuda, dtype=torch.bfloat16)
    ok = np.array([[4, 6], [0, 0], [1, 9]], dtype=np.int32)
    _regroup(torch.from_numpy(ok).to(cuda), A, B, 0, M, src, 1, 0, dst, status=status)
    assert _lib.moe_sync_status(status) == 0


@pytest.mark.parametrize("width,aux", [(256, 0), (7, 3), (512, 56)])
def test_exchange_pull_and_push_match_oracle(cuda, width, aux):
    from combine_moe_route_10_b200 import _lib
    from _ep_oracle_ops import OracleOps
    g = np.random.default_rng(width + aux)
    R, E, rank = 3, 6, 1
    C = g.integers(0, 30, size=(R, E)).astype(np.int32)
    C[2, 2:4] = 0                                   # source 2 sends this rank nothing
    cap = int(C.sum(axis=1).max()) + 4
    dt = torch.bfloat16 if width % 2 == 0 else torch.float32
    peers = [torch.randn(cap, width, device=cuda).to(dt) for _ in range(R)]
    peers_aux = [torch.randn(cap, aux, device=cuda) for _ in range(R)] if aux else None
    n_loc = int(C[:, 2:4].sum())
    local = torch.full((n_loc + 5, width), 3.0, device=cuda, dtype=dt)
    local_aux = torch.full((n_loc + 5, aux), -2.0, device=cuda) if aux else None
    offs = torch.full((3,), -7, dtype=torch.int32, device=cuda)
    status = torch.zeros(64, dtype=torch.int32, device=cuda)
    ac = torch.from_numpy(C.reshape(-1)).to(cuda)
    table = lambda ts: torch.tensor([t.data_ptr() for t in ts], dtype=torch.int64, device=cuda)
    rb = width * local.element_size()
    # expected: the same step on CPU copies with the oracle's layouts
    o = OracleOps()
    cpu_peers = [t.cpu() for t in peers]
    cpu_aux = [t.cpu() for t in peers_aux] if aux else None
    exp_local, exp_aux = local.cpu(), (local_aux.cpu() if aux else None)
    exp_offs = torch.zeros(3, dtype=torch.int32)
    o.exchange(ac.cpu(), R, E, rank, 0, cpu_peers, cpu_aux, cap, exp_local, exp_aux, exp_offs)
    _lib.moe_ep_exchange(ac, R, E, rank, _lib.MOE_EP_PULL, table(peers),
                         table(peers_aux) if aux else None, cap, local, local_aux,
                         local.shape[0], rb, aux * 4, offs, status)
    assert _lib.moe_sync_status(status) == 0
    assert torch.equal(local.cpu(), exp_local)
    assert torch.equal(offs.cpu(), exp_offs)
    if aux:
        assert torch.equal(local_aux.cpu(), exp_aux)
    # push the (new) local rows back into every source's buffer
    local2 = torch.randn(n_loc + 5, width, device=cuda).to(dt)
    o.exchange(ac.cpu(), R, E, rank, 1, cpu_peers, None, cap, local2.cpu(), None)
    _lib.moe_ep_exchange(ac, R, E, rank, _lib.MOE_EP_PUSH, table(peers), None, cap, local2, None,
                         local2.shape[0], rb, 0, None, status)
    assert _lib.moe_sync_status(status) == 0
    for s_ in range(R):
        assert torch.equal(peers[s_].cpu(), cpu_peers[s_]), s_


def test_exchange_rejects_counts_that_do_not_fit(cuda):
    from combine_moe_route_10_b200 import _lib
    R, E, rank, cap = 2, 4, 1, 10
    peers = [torch.zeros(cap, 64, device=cuda, dtype=torch.bfloat16) for _ in range(R)]
    table = torch.tensor([t.data_ptr() for t in peers], dtype=torch.int64, device=cuda)
    status = torch.zeros(64, dtype=torch.int32, device=cuda)
    for C in (np.array([[1, -1, 2, 2], [0, 0, 1, 1]]),   # a negative count before this rank's block
              np.array([[5, 4, 1, 1], [0, 0, 1, 1]]),    # source 0: block ends at row 11 > 10
              np.array([[0, 0, 9, 0], [0, 0, 0, 9]])):   # 18 rows into a 10-row local buffer
        local = torch.zeros(cap, 64, device=cuda, dtype=torch.bfloat16)
        peers[0].fill_(1.0)
        _lib.moe_ep_exchange(torch.from_numpy(C.astype(np.int32).reshape(-1)).to(cuda), R, E, rank,
                             _lib.MOE_EP_PULL, table, None, cap, local, None, cap, 128, 0, None,
                             status)
        assert _lib.moe_sync_status(status) == _lib.MOE_ERR_INVALID_COUNTS, C
        assert int(local.abs().sum().item()) == 0


def _single_device(w, d, R_total, payload):
    from combine_moe_route_10_b200 import MoeShuffle
    T = sum(t.shape[0] for t in d["x"])
    m = MoeShuffle(T, w.H, w.E, w.k, R_total, w.F, payload=payload)
    y = m.forward(torch.cat(d["logits"]).contiguous(), torch.cat(d["x"]).contiguous(),
                  d["w_gate"], d["w_up"], d["w_down"]).clone()
    assert m.status() == 0
    return y


def _ep_threads(w, d, R, payload, mode, steps=2):
    from combine_moe_route_10_b200.ep import MoeEP
    E_loc = w.E // R

    def rank(r, comm):
        sl = slice(r * E_loc, (r + 1) * E_loc)
        ep = MoeEP(d["x"][r].shape[0], w.H, w.E, w.k, w.F, comm=comm, payload=payload, mode=mode)
        for _ in range(steps):
            y = ep.forward(d["logits"][r], d["x"][r], d["w_gate"][sl].contiguous(),
                           d["w_up"][sl].contiguous(), d["w_down"][sl].contiguous())
        torch.cuda.synchronize()
        assert ep.status() == 0
        return y.clone(), ep

    return run_ranks(R, rank)


@pytest.mark.parametrize("name", ["tiny", "train-small", "finegrained-small", "decode-small"])
@pytest.mark.parametrize("mode", ["ht", "ll", "p2p"])
def test_four_emulated_ranks_equal_the_single_device_path(cuda, name, mode):
    R = 4
    w = mi.get(name)
    d = mi.make_ep_inputs(w, R, seed=2, device="cuda")
    y_ref = _single_device(w, d, R, w.payload)
    res = _ep_threads(w, d, R, w.payload, mode)
    for r in range(R):
        assert torch.equal(res[r][0], y_ref[r * w.T:(r + 1) * w.T]), (name, mode, r)


def test_emulated_ranks_meet_the_oracle_bar(cuda):
    R = 2
    w = mi.get("tiny")
    d = mi.make_ep_inputs(w, R, seed=4, device="cuda")
    res = _ep_threads(w, d, R, "bf16", "ht", steps=1)
    o = moe.pipeline(np.concatenate([np_(t) for t in d["logits"]]),
                     np.concatenate([bits16(t) for t in d["x"]]), bits16(d["w_gate"]),
                     bits16(d["w_up"]), bits16(d["w_down"]), w.k, R)
    y = np.concatenate([bits16(res[r][0]) for r in range(R)])
    # the expert rows of rank r are rows [rank_offsets[r], rank_offsets[r+1]) of the single-device
    # layout: compare them through the combine with the usual bar
    eo = np.zeros_like(o["expert_out"])
    h = np.zeros_like(o["h"])
    for r in range(R):
        ep = res[r][1]
        lo, hi = o["rank_offsets"][r], o["rank_offsets"][r + 1]
        n = hi - lo
        eo[lo:hi] = bits16(ep.expert_out)[:n]
        # the SwiGLU intermediate [rows, F] sits 256 bytes into the FFN workspace
        h[lo:hi] = bits16(ep.ws_ffn[256:256 + ep.cap * w.F * 2].view(torch.bfloat16)
                          .view(ep.cap, w.F))[:n]
    assert_ffn_and_combine(h, eo, y, o["h"], o["expert_out"], o["y"], o["expert_offsets"],
                           d["w_down"], o["slot_row"], o["topk_w"], "ep tiny")


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_nccl_one_rank_eager_and_graph(cuda):
    import torch.distributed as dist
    from combine_moe_route_10_b200.ep import MoeEP
    w = mi.get("train-small")
    d = mi.make_ep_inputs(w, 1, seed=6, device="cuda")
    y_ref = _single_device(w, d, 1, "bf16")
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0,
                            world_size=1, device_id=cuda)
    graphs = []
    try:
        for mode in ("ht", "ll", "p2p"):
            ep = MoeEP(w.T, w.H, w.E, w.k, w.F, mode=mode)
            y = ep.forward(d["logits"][0], d["x"][0], d["w_gate"], d["w_up"], d["w_down"])
            torch.cuda.synchronize()
            assert ep.status() == 0
            assert torch.equal(y, y_ref), mode
        d2 = mi.make_ep_inputs(w, 1, seed=8, device="cuda")
        d2["w_gate"], d2["w_up"], d2["w_down"] = d["w_gate"], d["w_up"], d["w_down"]
        y_ref2 = _single_device(w, d2, 1, "bf16")
        # the low-latency and peer-memory steps have no host synchronisation: capture them
        graphs = []
        for mode in ("ll", "p2p"):
            ep = MoeEP(w.T, w.H, w.E, w.k, w.F, mode=mode)
            logits = d["logits"][0].clone()
            x = d["x"][0].clone()
            ep.forward(logits, x, d["w_gate"], d["w_up"], d["w_down"])
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            graphs.append(g)
            s = torch.cuda.Stream()
            s.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(s):
                with torch.cuda.graph(g, capture_error_mode="thread_local"):
                    ep.forward(logits, x, d["w_gate"], d["w_up"], d["w_down"])
            torch.cuda.current_stream().wait_stream(s)
            ep.y.zero_()
            g.replay()
            torch.cuda.synchronize()
            assert torch.equal(ep.y, y_ref), mode
            # new inputs written into the captured tensors
            logits.copy_(d2["logits"][0])
            x.copy_(d2["x"][0])
            g.replay()
            torch.cuda.synchronize()
            assert torch.equal(ep.y, y_ref2), mode
    finally:
        graphs = None
        g = None
        torch.cuda.synchronize()
        dist.destroy_process_group()


def test_nccl_one_rank_peer_mode_through_symmetric_memory(cuda):
    """The peer buffers of the p2p mode through torch symmetric memory (the mapping used between
    GPUs), at one rank."""
    import torch.distributed as dist
    from combine_moe_route_10_b200.ep import MoeEP, TorchComm
    w = mi.get("finegrained-small")
    d = mi.make_ep_inputs(w, 1, seed=9, device="cuda")
    y_ref = _single_device(w, d, 1, "fp8")
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0,
                            world_size=1, device_id=cuda)
    try:
        ep = MoeEP(w.T, w.H, w.E, w.k, w.F, comm=TorchComm(symmetric=True), payload="fp8",
                   mode="p2p")
        for _ in range(2):
            y = ep.forward(d["logits"][0], d["x"][0], d["w_gate"], d["w_up"], d["w_down"])
        torch.cuda.synchronize()
        assert ep.status() == 0
        assert torch.equal(y, y_ref)
        del ep
    finally:
        torch.cuda.synchronize()
        dist.destroy_process_group()


@pytest.mark.parametrize("name", ["tiny", "train-small", "finegrained-small"])
@pytest.mark.parametrize("mode", ["ht", "ll", "p2p"])
def test_four_emulated_ranks_backward_equals_the_single_device_backward(cuda, name, mode):
    """MoeEP.backward over 4 thread ranks on one GPU: dx, d_logits and d_topk_w of every rank and
    the weight gradients of its experts equal MoeShuffle.backward over all ranks' tokens, bit for
    bit (every row meets the same kernels in the same order)."""
    from combine_moe_route_10_b200 import MoeShuffle
    from combine_moe_route_10_b200.ep import MoeEP
    R = 4
    w = mi.get(name)
    d = mi.make_ep_inputs(w, R, seed=12, device="cuda")
    g = torch.Generator(device="cuda").manual_seed(13)
    dys = [torch.randn((w.T, w.H), generator=g, device="cuda").to(torch.bfloat16)
           for _ in range(R)]
    T = R * w.T
    single = MoeShuffle(T, w.H, w.E, w.k, R, w.F, payload=w.payload)
    logits = torch.cat(d["logits"]).contiguous()
    single.forward(logits, torch.cat(d["x"]).contiguous(), d["w_gate"], d["w_up"], d["w_down"])
    ref = single.backward(torch.cat(dys).contiguous(), logits, d["w_gate"], d["w_up"],
                          d["w_down"])
    torch.cuda.synchronize()
    assert single.status() == 0
    E_loc = w.E // R

    def rank(r, comm):
        sl = slice(r * E_loc, (r + 1) * E_loc)
        wts = [d[key][sl].contiguous() for key in ("w_gate", "w_up", "w_down")]
        ep = MoeEP(w.T, w.H, w.E, w.k, w.F, comm=comm, payload=w.payload, mode=mode)
        ep.forward(d["logits"][r], d["x"][r], *wts)
        gr = ep.backward(dys[r], d["logits"][r], *wts)
        torch.cuda.synchronize()
        assert ep.status() == 0
        return {key: v.clone() for key, v in gr.items()}

    res = run_ranks(R, rank)
    for r in range(R):
        ts = slice(r * w.T, (r + 1) * w.T)
        es = slice(r * E_loc, (r + 1) * E_loc)
        for key in ("dx", "d_logits", "d_topk_w"):
            assert torch.equal(res[r][key], ref[key][ts]), (name, mode, r, key)
        for key in ("d_w_gate", "d_w_up", "d_w_down"):
            assert torch.equal(res[r][key], ref[key][es]), (name, mode, r, key)
