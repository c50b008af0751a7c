"""Brute force on tiny inputs: an independent dictionary-based restatement of the whole path."""
import math

import numpy as np
import pytest

from oracle import moe
from oracle.numerics import bf16_bits, bf16_from_bits, bf16_round


def restated(logits, x, wg, wu, wd, k, R, cap):
    T, E = logits.shape
    H = x.shape[1]
    # route: sort (value desc, id asc)
    picks = []
    for t in range(T):
        order = sorted(range(E), key=lambda e: (-float(logits[t, e]), e))[:k]
        m = float(logits[t, order[0]])
        ex = [math.exp(float(logits[t, e]) - m) for e in order]
        picks.append([(e, np.float32(v / sum(ex))) for e, v in zip(order, ex)])
    # dispatch: per-expert lists in token order, then truncation to the capacity
    lists = {e: [] for e in range(E)}
    for t in range(T):
        for j, (e, _) in enumerate(picks[t]):
            lists[e].append((t, j))
    kept = {e: (lst if cap == 0 else lst[:cap]) for e, lst in lists.items()}
    where = {}
    rows = []
    for e in range(E):
        for (t, j) in kept[e]:
            where[(t, j)] = len(rows)
            rows.append((e, t))
    # FFN per row
    X = bf16_from_bits(x).astype(np.float64)
    outs = []
    for e, t in rows:
        G = [float(np.dot(X[t], bf16_from_bits(wg[e, f]).astype(np.float64))) for f in range(wg.shape[1])]
        U = [float(np.dot(X[t], bf16_from_bits(wu[e, f]).astype(np.float64))) for f in range(wg.shape[1])]
        h = [float(bf16_round(gv / (1 + math.exp(-gv)) * uv)) for gv, uv in zip(G, U)]
        outs.append([float(bf16_round(np.dot(h, bf16_from_bits(wd[e, o]).astype(np.float64))))
                     for o in range(H)])
    # combine, fp32 in slot order
    y = np.zeros((T, H), dtype=np.float32)
    for t in range(T):
        for j, (e, wt) in enumerate(picks[t]):
            if (t, j) in where:
                y[t] = y[t] + np.float32(wt) * np.array(outs[where[(t, j)]], dtype=np.float32)
    return picks, where, rows, bf16_bits(y)


@pytest.mark.parametrize("T,E,k,R,cap", [(1, 1, 1, 1, 0), (5, 4, 2, 2, 0), (8, 8, 3, 4, 2),
                                         (6, 3, 3, 1, 0), (7, 8, 8, 8, 3), (8, 4, 1, 4, 1)])
def test_tiny_pipeline_matches_restatement(T, E, k, R, cap):
    g = np.random.default_rng(100 + T * E + k)
    H, F = 16, 8
    logits = g.normal(size=(T, E)).astype(np.float32)
    x = bf16_bits(g.normal(size=(T, H)))
    wg, wu = bf16_bits(g.normal(0, 0.3, (E, F, H))), bf16_bits(g.normal(0, 0.3, (E, F, H)))
    wd = bf16_bits(g.normal(0, 0.3, (E, H, F)))
    o = moe.pipeline(logits, x, wg, wu, wd, k, R)
    if cap:
        p = moe.dispatch_plan(o["topk_idx"], E, R, cap)
        send, _ = moe.dispatch_payload(x, p)
        _, ye = moe.expert_ffn(bf16_from_bits(send).astype(np.float64), p["expert_offsets"], wg, wu, wd)
        o = dict(o, **p, expert_out=ye, y=moe.combine(ye, p["slot_row"], o["topk_w"], T, H))
    picks, where, rows, y = restated(logits, x, wg, wu, wd, k, R, cap)
    assert [[e for e, _ in p] for p in picks] == o["topk_idx"].tolist()
    assert np.allclose([[w for _, w in p] for p in picks], o["topk_w"], rtol=1e-6)
    for t in range(T):
        for j in range(k):
            assert o["slot_row"][t, j] == where.get((t, j), -1)
    assert [t for _, t in rows] == o["row_token"].tolist()
    assert np.array_equal(y, o["y"])
