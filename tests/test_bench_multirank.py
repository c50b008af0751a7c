"""The multi-GPU path of bench.py (independent replicas, max over ranks) on CPU with gloo ranks."""
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import moe_inputs as mi


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        local_ms = 10.0 * (rank + 1)                       # rank 1 is the slower one
        agg = bench.aggregate(local_ms, tokens_per_rank=128, steps=5, device="cpu")
        # replicas draw different inputs (seed = rank)
        d = mi.make_inputs(mi.get("tiny"), seed=rank, device="cpu", weights=False)
        out[rank] = (agg["value"], agg["ms_per_step"], agg["n_ranks"], float(d["logits"][0, 0]))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_rank():
    world, port = 2, _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.start_processes(_rank_main, args=(world, port, out), nprocs=world, join=True,
                           start_method="spawn")
        res = dict(out)
    assert set(res) == {0, 1}
    for rank in range(world):
        value, ms_per_step, n, _ = res[rank]
        assert n == 2
        assert ms_per_step == pytest.approx(20.0 / 5)      # the max over ranks, per step
        assert value == pytest.approx(2 * 128 * 5 / 0.020)  # both ranks' tokens / slowest time
    assert res[0][3] != res[1][3]


def test_single_process_aggregate():
    agg = bench.aggregate(8.0, tokens_per_rank=100, steps=4, device="cpu")
    assert agg["n_ranks"] == 1 and agg["ms_per_step"] == 2.0
    assert agg["value"] == pytest.approx(400 / 0.008)
