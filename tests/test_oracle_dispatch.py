"""Pins of the oracle dispatch: printed capacity example, bijection, token order, drop rule, FP8."""
import os

import numpy as np
import pytest

from oracle import moe
from oracle.numerics import bf16_from_bits, e4m3_decode

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_capacity_printed_example():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "capacity_example.txt"))
            if l.strip() and not l.startswith("#")]
    assert rows
    for cf, T, k, E, want in rows:
        assert moe.capacity(float(cf), int(T), int(k), int(E)) == int(want)


def test_capacity_rounding_and_no_limit():
    assert moe.capacity(1.25, 16384, 2, 128) == 320
    assert moe.capacity(1.0, 10, 1, 3) == 4          # ceil(10/3)
    assert moe.capacity(0.0, 100, 2, 8) == 0


def random_idx(g, T, E, k, hot=None):
    keys = g.random((T, E))
    if hot is not None:
        keys[:, hot] += 0.7
    return np.argsort(-keys, axis=1)[:, :k].astype(np.int32)


@pytest.mark.parametrize("T,E,k,R,cap", [(40, 8, 2, 4, 0), (64, 16, 4, 8, 0), (100, 8, 2, 2, 7),
                                         (33, 4, 4, 1, 5), (50, 8, 3, 8, 1)])
def test_plan_invariants(T, E, k, R, cap):
    g = np.random.default_rng(T + E + k)
    idx = random_idx(g, T, E, k, hot=0)
    p = moe.dispatch_plan(idx, E, R, cap)
    S, sr, rt, off = p["S"], p["slot_row"], p["row_token"], p["expert_offsets"]
    routed = np.bincount(idx.ravel(), minlength=E)
    assert np.array_equal(p["expert_routed"], routed)
    assert routed.sum() == T * k
    kept = np.minimum(routed, cap) if cap else routed
    assert np.array_equal(p["expert_counts"], kept)
    assert off[0] == 0 and np.all(np.diff(off) == kept) and off[E] == S
    assert np.array_equal(p["rank_offsets"], off[np.arange(R + 1) * (E // R)])
    kept_rows = sr[sr >= 0]
    assert np.array_equal(np.sort(kept_rows), np.arange(S))      # bijection onto [0, S)
    for t in range(T):
        for j in range(k):
            e = idx[t, j]
            earlier = int(np.sum(idx[:t] == e))                  # brute-force position
            if cap and earlier >= cap:
                assert sr[t, j] == -1
            else:
                assert sr[t, j] == off[e] + earlier
                assert rt[sr[t, j]] == t
    for e in range(E):
        seg = rt[off[e]:off[e + 1]]
        assert np.all(np.diff(seg) > 0)                          # ascending token order


def test_out_of_range_ids_rejected():
    with pytest.raises(ValueError):
        moe.dispatch_plan(np.array([[0, 8]]), 8, 1, 0)


def test_bf16_payload_bytes():
    g = np.random.default_rng(9)
    T, H, E, k = 30, 64, 8, 2
    x = g.integers(0, 2 ** 16, (T, H), dtype=np.uint16)
    p = moe.dispatch_plan(random_idx(g, T, E, k), E, 2, 0)
    send, sc = moe.dispatch_payload(x, p)
    assert sc is None
    for row in range(p["S"]):
        assert np.array_equal(send[row], x[p["row_token"][row]])


def test_fp8_payload_scale_and_error_bound():
    g = np.random.default_rng(10)
    T, H, E, k = 20, 256, 4, 2
    xf = g.normal(size=(T, H)).astype(np.float32)
    xf[3, :128] = 0.0                                            # an all-zero block: scale 1
    xf[4, 5] = 1e-30                                             # underflows to bf16 subnormal/0
    x = (xf.view(np.uint32) >> 16).astype(np.uint16)             # truncation: any bf16 pattern
    xv = bf16_from_bits(x).astype(np.float64)
    p = moe.dispatch_plan(random_idx(g, T, E, k), E, 1, 0)
    send, sc = moe.dispatch_payload(x, p, fp8=True)
    assert send.dtype == np.uint8 and sc.shape == (p["S"], H // 128)
    for row in range(p["S"]):
        t = p["row_token"][row]
        for b in range(H // 128):
            blk = xv[t, b * 128:(b + 1) * 128]
            amax = np.max(np.abs(blk))
            s = sc[row, b]
            if amax == 0:
                assert s == 1.0 and np.all(send[row, b * 128:(b + 1) * 128] == 0)
                continue
            assert s == np.float32(amax) / np.float32(448.0)
            q = e4m3_decode(send[row, b * 128:(b + 1) * 128]) * np.float64(s)
            # the largest element lands on the top code
            assert np.max(np.abs(e4m3_decode(send[row, b * 128:(b + 1) * 128]))) == 448.0
            # round to nearest with 3 fraction bits: relative error <= 2^-4 for normals,
            # absolute error <= 2^-10 * scale in the subnormal range
            err = np.abs(q - blk)
            assert np.all(err <= np.maximum(2.0 ** -4 * np.abs(blk), 2.0 ** -10 * s) * (1 + 1e-6))
