"""Expert parallelism over real process groups on CPU: gloo ranks run ``MoeEP`` (count exchange,
split sizes, padded low-latency blocks, regrouping, the return trip) with oracle-backed local steps,
and every rank's output must equal, bit for bit, its slice of the single-device oracle over all
ranks' tokens."""
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import moe_inputs as mi
from oracle import moe
from oracle.numerics import bf16_bits


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


T_RANK = 40  # tokens per rank (the fp64 FFN stays quick)


def _inputs(R, payload):
    w = mi.get("tiny")
    d = mi.make_ep_inputs(w, R, seed=5)
    lg = [t[:T_RANK].contiguous() for t in d["logits"]]
    xs = [t[:T_RANK].contiguous() for t in d["x"]]
    # rank 0's tokens never pick the last rank's experts: a zero-row block in every exchange
    E_loc = w.E // R
    lg[0][:, w.E - E_loc:] -= 50.0
    return w, lg, xs, d


def _rank_main(rank, world, port, out):
    from combine_moe_route_10_b200.ep import MoeEP, TorchComm
    from _ep_oracle_ops import OracleOps
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        res = {}
        for payload in ("bf16", "fp8"):
            w, lg, xs, d = _inputs(world, payload)
            E_loc = w.E // world
            sl = slice(rank * E_loc, (rank + 1) * E_loc)
            for mode, recv_rows in (("ht", 8), ("ll", None)):      # ht starts small and grows
                ops = OracleOps()
                ep = MoeEP(T_RANK, w.H, w.E, w.k, w.F, comm=TorchComm(), payload=payload,
                           mode=mode, recv_rows=recv_rows, device="cpu", ops=ops)
                for _ in range(2):                                  # a second step reuses buffers
                    y = ep.forward(lg[rank], xs[rank], d["w_gate"][sl].contiguous(),
                                   d["w_up"][sl].contiguous(), d["w_down"][sl].contiguous())
                res[(payload, mode)] = (y.view(torch.int16).numpy().view(np.uint16).copy(),
                                        ops.calls.count("regroup") // 2)
        out[rank] = res
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_gloo_ranks_match_the_single_device_oracle(world):
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.start_processes(_rank_main, args=(world, port, out), nprocs=world, join=True,
                           start_method="spawn")
        res = dict(out)
    assert set(res) == set(range(world))
    for payload in ("bf16", "fp8"):
        w, lg, xs, d = _inputs(world, payload)
        wb = [bf16_bits(d[key].float().numpy()) for key in ("w_gate", "w_up", "w_down")]
        ref = moe.pipeline(np.concatenate([a.numpy() for a in lg]),
                           np.concatenate([bf16_bits(a.float().numpy()) for a in xs]), *wb, w.k,
                           world, fp8=payload == "fp8")["y"]
        for mode, regroups in (("ht", 2), ("ll", 4)):
            for r in range(world):
                y, n_regroup = res[r][(payload, mode)]
                assert n_regroup == regroups, (payload, mode)
                assert np.array_equal(y, ref[r * T_RANK:(r + 1) * T_RANK]), (payload, mode, r)


def test_thread_loopback_matches_the_oracle_too():
    """The in-process R-rank emulation used by the single-GPU tests gives the same results, and
    runs the peer-memory mode (one address space) as well."""
    from combine_moe_route_10_b200.ep import MoeEP
    from _ep_loopback import run_ranks
    from _ep_oracle_ops import OracleOps
    R = 4
    w, lg, xs, d = _inputs(R, "bf16")
    E_loc = w.E // R

    def rank(r, comm):
        sl = slice(r * E_loc, (r + 1) * E_loc)
        out = {}
        for mode in ("ht", "ll", "p2p"):
            ep = MoeEP(T_RANK, w.H, w.E, w.k, w.F, comm=comm, payload=payload, mode=mode,
                       device="cpu", ops=OracleOps())
            for _ in range(2):
                y = ep.forward(lg[r], xs[r], d["w_gate"][sl].contiguous(),
                               d["w_up"][sl].contiguous(), d["w_down"][sl].contiguous())
            out[mode] = y.view(torch.int16).numpy().view(np.uint16).copy()
        return out

    for payload in ("bf16", "fp8"):
        w, lg, xs, d = _inputs(R, payload)
        res = run_ranks(R, rank)
        wb = [bf16_bits(d[key].float().numpy()) for key in ("w_gate", "w_up", "w_down")]
        ref = moe.pipeline(np.concatenate([a.numpy() for a in lg]),
                           np.concatenate([bf16_bits(a.float().numpy()) for a in xs]), *wb, w.k,
                           R, fp8=payload == "fp8")["y"]
        for r in range(R):
            for mode in ("ht", "ll", "p2p"):
                assert np.array_equal(res[r][mode], ref[r * T_RANK:(r + 1) * T_RANK]), \
                    (payload, mode, r)


def _dying_rank_main(rank, world, port, out):
    import datetime
    from combine_moe_route_10_b200.ep import MoeEP, TorchComm
    from _ep_oracle_ops import OracleOps
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=5))
    w, lg, xs, d = _inputs(world, "bf16")
    E_loc = w.E // world
    sl = slice(rank * E_loc, (rank + 1) * E_loc)
    ep = MoeEP(T_RANK, w.H, w.E, w.k, w.F, comm=TorchComm(), mode="ht", device="cpu",
               ops=OracleOps())
    if rank == world - 1:
        out[rank] = "left"
        return  # leaves between steps: never joins the exchange (its group is torn down at exit)
    try:
        ep.forward(lg[rank], xs[rank], d["w_gate"][sl].contiguous(), d["w_up"][sl].contiguous(),
                   d["w_down"][sl].contiguous())
        out[rank] = "no error"
    except Exception as e:  # the collective ends with an error instead of waiting for good
        out[rank] = f"error: {type(e).__name__}"


def test_a_rank_that_leaves_ends_the_others_collectives_with_an_error():
    """A rank that leaves before the exchange: the other ranks' next collective ends with an error
    within the process group's timeout (a host-side failure; no device is involved)."""
    world, port = 4, _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        ctx = mp.start_processes(_dying_rank_main, args=(world, port, out), nprocs=world,
                                 join=False, start_method="spawn")
        import time
        t0 = time.time()
        while not ctx.join(timeout=1):
            assert time.time() - t0 < 120, "ranks did not finish"
        res = dict(out)
    assert res[world - 1] == "left"
    for r in range(world - 1):
        assert res[r].startswith("error"), (r, res[r])


def test_thread_ranks_backward_matches_the_single_device_oracle():
    """MoeEP.backward over 4 thread ranks (oracle-backed steps), all three exchange modes and both
    payloads: every rank's dx, d_logits and d_topk_w and its experts' weight gradients equal the
    single-device oracle's backward over all ranks' tokens, bit for bit."""
    from combine_moe_route_10_b200.ep import MoeEP
    from _ep_loopback import run_ranks
    from _ep_oracle_ops import OracleOps
    R = 4
    for payload in ("bf16", "fp8"):
        w, lg, xs, d = _inputs(R, payload)
        E_loc = w.E // R
        g = torch.Generator().manual_seed(3)
        dys = [torch.randn((T_RANK, w.H), generator=g).to(torch.bfloat16) for _ in range(R)]

        def rank(r, comm):
            sl = slice(r * E_loc, (r + 1) * E_loc)
            wts = [d[key][sl].contiguous() for key in ("w_gate", "w_up", "w_down")]
            out = {}
            for mode in ("ht", "ll", "p2p"):
                ep = MoeEP(T_RANK, w.H, w.E, w.k, w.F, comm=comm, payload=payload, mode=mode,
                           device="cpu", ops=OracleOps())
                ep.forward(lg[r], xs[r], *wts)
                gr = ep.backward(dys[r], lg[r], *wts)
                out[mode] = {key: v.clone() for key, v in gr.items()}
            return out

        res = run_ranks(R, rank)
        wb = [bf16_bits(d[key].float().numpy()) for key in ("w_gate", "w_up", "w_down")]
        fwd = moe.pipeline(np.concatenate([a.numpy() for a in lg]),
                           np.concatenate([bf16_bits(a.float().numpy()) for a in xs]), *wb, w.k, R,
                           fp8=payload == "fp8")
        ref = moe.backward(fwd, np.concatenate([bf16_bits(a.float().numpy()) for a in dys]),
                           np.concatenate([a.numpy() for a in lg]), *wb, fp8=payload == "fp8")
        for r in range(R):
            ts = slice(r * T_RANK, (r + 1) * T_RANK)
            es = slice(r * E_loc, (r + 1) * E_loc)
            for mode in ("ht", "ll", "p2p"):
                got = res[r][mode]
                what = (payload, mode, r)
                assert np.array_equal(got["dx"].view(torch.int16).numpy().view(np.uint16),
                                      ref["dx"][ts]), what
                assert np.array_equal(got["d_logits"].numpy(), ref["d_logits"][ts]), what
                assert np.array_equal(got["d_topk_w"].numpy(), ref["d_w"][ts]), what
                for key in ("d_w_gate", "d_w_up", "d_w_down"):
                    assert np.array_equal(got[key].numpy(), ref[key][es]), (what, key)
