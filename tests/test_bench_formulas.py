"""The benchmark's roofline arithmetic: algorithmic bytes and flops per stage, checked against the
per-configuration figures worked out by hand from the stage definitions (dispatch reads each token
row once and writes each kept row once; the combine reads each kept row once and writes each token
row once; the FFN moves the active experts' weights once and does 6 S H F flops)."""
import bench
import moe_inputs as mi

MB, GB = 1e6, 1e9


def close(a, b, rel):
    return abs(a - b) <= rel * abs(b)


def test_train_dispatch_and_combine_bytes():
    w = mi.get("train")
    S = w.T * w.k
    a = bench.algorithmic(w, S, w.E)
    # 4096 x 4096 bf16 read (33.6 MB) + 8192 x 4096 bf16 written (67.1 MB), plus index arrays
    assert close(a["dispatch"], 100.7 * MB, 0.005)
    assert close(a["combine"], 100.7 * MB, 0.005)
    assert a["ffn_flops"] == 6 * 8192 * 4096 * 14336          # 2.89 TFLOP
    assert a["ffn_weight_bytes"] == 8 * 3 * 4096 * 14336 * 2  # 2.82 GB


def test_finegrained_fp8_bytes():
    w = mi.get("finegrained")
    S = w.T * w.k
    a = bench.algorithmic(w, S, w.E)
    # 58.7 MB of bf16 rows read; 234.9 MB of e4m3 codes + 7.3 MB of fp32 scales written
    assert close(a["dispatch"], 301 * MB, 0.005)
    # 469.8 MB of bf16 expert outputs read, 58.7 MB written
    assert close(a["combine"], 528.5 * MB, 0.005)
    assert close(a["ffn_weight_bytes"], 22.5 * GB, 0.005)
    # the FFN's method bytes: the codes and scales as dispatched, read once, and bf16 outputs
    # written once; the bf16 intermediate and the dequantised rows are the implementation's own
    assert a["ffn_bytes"] == a["ffn_weight_bytes"] + S * w.H + S * (w.H // 128) * 4 + S * w.H * 2
    assert a["ffn_impl_overhead"] == 2 * S * w.F * 2 + 4 * S * w.H


def test_decode_and_skewed_ffn_figures():
    d = mi.get("decode")
    a = bench.algorithmic(d, d.T * d.k, d.E)
    assert close(a["ffn_flops"], 90.2e9, 0.001)
    assert close(a["ffn_weight_bytes"], 2.82 * GB, 0.001)
    s = mi.get("skewed")
    a = bench.algorithmic(s, 20488, s.E)
    assert close(a["ffn_weight_bytes"], 11.3 * GB, 0.005)
    # bytes scale with the kept rows only (dropped slots are neither written nor read)
    b = bench.algorithmic(s, 20488 + 1000, s.E)
    assert b["dispatch"] - a["dispatch"] == 1000 * (s.H * 2 + 4)
    assert b["combine"] - a["combine"] == 1000 * s.H * 2


def test_recorded_traffic_is_near_the_algorithmic_bytes():
    """The DRAM traffic recorded from ncu captures lies between 0.95x and 1.3x the algorithmic FFN
    bytes plus the implementation's own overhead, for the same workload (active experts and kept
    rows from the oracle's routing)."""
    import numpy as np
    from oracle import moe
    assert set(bench.FFN_TRAFFIC) <= set(mi.WORKLOADS)
    for name, t in bench.FFN_TRAFFIC.items():
        w = mi.get(name)
        d = mi.make_inputs(w, seed=0, device="cpu", weights=False)
        idx, _, _ = moe.route(d["logits"].numpy(), w.k)
        plan = moe.dispatch_plan(idx, w.E, w.R, moe.capacity(w.capacity_factor, w.T, w.k, w.E))
        active = int((np.diff(plan["expert_offsets"]) > 0).sum())
        a = bench.algorithmic(w, plan["S"], active)
        alg = a["ffn_bytes"] + a["ffn_impl_overhead"]
        assert 0.95 * alg <= t <= 1.3 * alg, (name, t / alg)
