"""Brute force on tiny inputs: an independent dictionary-based restatement of the whole path.

The restatement uses Python floats and lists, sorted() for the top-k, and for the FP8 payload the
e4m3 value table and bf16 cast of torch (not the oracle's number-format code): per 128-element
block, scale = fp32(amax / 448) and q = fp32(x / scale) (a double-precision quotient rounded once to
fp32 equals the IEEE fp32 quotient, since 53 >= 2 * 24 + 2), the nearest e4m3 value with ties to
the even code and saturation at 448, then x = bf16(fp32(value * scale)).
"""
import math

import numpy as np
import pytest
import torch

from oracle import moe
from oracle.numerics import bf16_bits, bf16_from_bits, bf16_round

_E4M3_VALUES = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn) \
    .to(torch.float64).tolist()
_E4M3_FINITE = [(c, v) for c, v in enumerate(_E4M3_VALUES) if not math.isnan(v)]


def restated_fp8_token(row):
    """Dequantised FFN input values of one token row (list of Python floats) under the FP8 payload."""
    out = []
    for b0 in range(0, len(row), 128):
        blk = row[b0:b0 + 128]
        amax = max(abs(v) for v in blk)
        scale = 1.0 if amax == 0 else float(np.float32(amax / 448.0))
        for v in blk:
            qv = float(np.float32(v / scale))
            if abs(qv) >= 448.0:
                code = 0x7E if qv > 0 else 0xFE
            else:
                best = min(_E4M3_FINITE, key=lambda cv: (abs(qv - cv[1]), cv[0] & 1))
                code = best[0]
                if best[1] == 0.0:
                    code = 0x80 if math.copysign(1.0, qv) < 0 else 0x00
            prod = float(np.float32(_E4M3_VALUES[code] * scale))   # exact product, one fp32 rounding
            out.append(float(torch.tensor(prod, dtype=torch.float32).to(torch.bfloat16).item()))
    return out


def restated(logits, x, wg, wu, wd, k, R, cap, fp8=False, renormalize=True):
    T, E = logits.shape
    H = x.shape[1]
    # route: sort (value desc, id asc); weights over the selected k, or over all E
    picks = []
    for t in range(T):
        order = sorted(range(E), key=lambda e: (-float(logits[t, e]), e))[:k]
        m = float(logits[t, order[0]])
        ex = [math.exp(float(logits[t, e]) - m) for e in order]
        den = sum(ex) if renormalize else sum(math.exp(float(logits[t, e]) - m) for e in range(E))
        picks.append([(e, np.float32(v / den)) for e, v in zip(order, ex)])
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
    # FFN per row (for FP8, on the token's quantised-then-dequantised values)
    X = bf16_from_bits(x).astype(np.float64)
    if fp8:
        X = np.array([restated_fp8_token(X[t].tolist()) for t in range(T)])
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


@pytest.mark.parametrize("T,E,k,R,cap,renorm", [(4, 4, 2, 2, 0, True), (8, 8, 3, 4, 2, True),
                                               (6, 3, 3, 1, 0, False), (7, 8, 8, 8, 3, False)])
def test_tiny_fp8_pipeline_matches_restatement(T, E, k, R, cap, renorm):
    g = np.random.default_rng(300 + T * E + k)
    H, F = 256, 8
    logits = g.normal(size=(T, E)).astype(np.float32)
    xf = g.normal(size=(T, H))
    xf[0, :128] = 0.0                                    # an all-zero block: scale 1
    xf[1, 128:] *= 1e-39                                 # a block with a subnormal scale
    xf[2, :128] = np.where(np.arange(128) % 2, -1e-6, 9.0)   # negatives that quantise to -0
    x = bf16_bits(xf)
    wg, wu = bf16_bits(g.normal(0, 0.1, (E, F, H))), bf16_bits(g.normal(0, 0.1, (E, F, H)))
    wd = bf16_bits(g.normal(0, 0.3, (E, H, F)))
    o = moe.pipeline(logits, x, wg, wu, wd, k, R, fp8=True, renormalize=renorm,
                     cf=0.0 if cap == 0 else cap * E / (T * k) - 1e-9)
    assert o["cap"] == cap
    picks, where, rows, y = restated(logits, x, wg, wu, wd, k, R, cap, fp8=True,
                                     renormalize=renorm)
    assert [[e for e, _ in p] for p in picks] == o["topk_idx"].tolist()
    assert np.allclose([[w for _, w in p] for p in picks], o["topk_w"], rtol=1e-6)
    for t in range(T):
        for j in range(k):
            assert o["slot_row"][t, j] == where.get((t, j), -1)
    assert [t for _, t in rows] == o["row_token"].tolist()
    assert np.array_equal(y, o["y"])
