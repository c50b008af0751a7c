"""Pins of the oracle FFN and combine: dense SwiGLU by triple loop, closed forms, sum order."""
import math

import numpy as np
import torch

from oracle import moe
from oracle.numerics import bf16_bits, bf16_from_bits, bf16_round


def rand_bf16(g, shape, std=1.0):
    return bf16_bits(g.normal(0, std, shape))


def test_single_expert_is_dense_swiglu_triple_loop():
    g = np.random.default_rng(11)
    rows, H, F = 3, 8, 6
    x = rand_bf16(g, (rows, H))
    wg, wu, wd = rand_bf16(g, (1, F, H), 0.5), rand_bf16(g, (1, F, H), 0.5), rand_bf16(g, (1, H, F), 0.5)
    off = np.array([0, rows], dtype=np.int32)
    h, y = moe.expert_ffn(bf16_from_bits(x).astype(np.float64), off, wg, wu, wd)
    X, WG, WU, WD = (bf16_from_bits(a).astype(np.float64).tolist() for a in (x, wg[0], wu[0], wd[0]))
    for r in range(rows):
        hr = []
        for f in range(F):
            gsum = sum(X[r][i] * WG[f][i] for i in range(H))
            usum = sum(X[r][i] * WU[f][i] for i in range(H))
            hr.append(float(bf16_round(gsum / (1 + math.exp(-gsum)) * usum)))
        for o in range(H):
            ysum = sum(hr[f] * WD[o][f] for f in range(F))
            assert y[r, o] == bf16_bits(ysum), (r, o)
        assert np.array_equal(h[r], bf16_bits(np.array(hr)))


def test_single_expert_matches_torch_matmul_fp64():
    g = np.random.default_rng(12)
    rows, H, F = 40, 64, 96
    x = rand_bf16(g, (rows, H))
    wg, wu, wd = (rand_bf16(g, s, 0.1) for s in [(1, F, H), (1, F, H), (1, H, F)])
    h, y = moe.expert_ffn(bf16_from_bits(x).astype(np.float64), np.array([0, rows]), wg, wu, wd)
    t = lambda a: torch.from_numpy(bf16_from_bits(a).astype(np.float64))
    G, U = t(x) @ t(wg[0]).T, t(x) @ t(wu[0]).T
    Hm = torch.nn.functional.silu(G) * U
    hb = torch.from_numpy(bf16_round(Hm.numpy()))
    Y = hb @ t(wd[0]).T
    assert np.array_equal(h, bf16_bits(hb.numpy()))
    assert np.array_equal(y, bf16_bits(Y.numpy()))


def test_identity_weights_closed_form_silu():
    # W_gate = W_up = W_down = I: h = bf16(silu(x) * x), y = h
    g = np.random.default_rng(13)
    n = 16
    x = rand_bf16(g, (5, n), 2.0)
    eye = bf16_bits(np.eye(n))[None]
    h, y = moe.expert_ffn(bf16_from_bits(x).astype(np.float64), np.array([0, 5]), eye, eye, eye)
    xv = bf16_from_bits(x).astype(np.float64)
    want = bf16_bits(xv * xv / (1 + np.exp(-xv)))
    assert np.array_equal(h, want) and np.array_equal(y, want)


def test_rows_use_their_own_expert():
    g = np.random.default_rng(14)
    E, H, F = 3, 16, 8
    x = rand_bf16(g, (7, H))
    w = [rand_bf16(g, s, 0.3) for s in [(E, F, H), (E, F, H), (E, H, F)]]
    off = np.array([0, 2, 2, 7])                         # expert 1 is empty
    _, y = moe.expert_ffn(bf16_from_bits(x).astype(np.float64), off, *w)
    for e, (lo, hi) in enumerate([(0, 2), (2, 2), (2, 7)]):
        if lo == hi:
            continue
        _, ye = moe.expert_ffn(bf16_from_bits(x[lo:hi]).astype(np.float64), np.array([0, hi - lo]),
                               w[0][e:e + 1], w[1][e:e + 1], w[2][e:e + 1])
        assert np.array_equal(y[lo:hi], ye)


def test_combine_identity_experts_return_input():
    g = np.random.default_rng(15)
    T, H, E, k = 64, 128, 8, 2
    l = g.normal(size=(T, E)).astype(np.float32)
    x = rand_bf16(g, (T, H))
    idx, w, _ = moe.route(l, k)
    p = moe.dispatch_plan(idx, E, 4, 0)
    send, _ = moe.dispatch_payload(x, p)
    y = moe.combine(send, p["slot_row"], w, T, H)        # expert_out = send (identity experts)
    xv = bf16_from_bits(x).astype(np.float64)
    yv = bf16_from_bits(y).astype(np.float64)
    ulp = 2.0 ** (np.floor(np.log2(np.abs(xv))) - 7)
    assert np.all(np.abs(yv - xv) <= ulp)
    assert np.mean(yv == xv) > 0.95


def test_combine_dropped_token_is_zero_and_sum_order():
    H = 8
    one = bf16_bits(np.ones((1, H)))
    eo = np.repeat(one, 4, axis=0)
    # slot order j = 0..3 in fp32: ((1 + 2^-8) + 2^-24) + 2^-24 stays 1 + 2^-8, a bf16 tie -> 1.0;
    # the reverse order would reach 1 + 2^-8 + 2^-23 and round up to 1 + 2^-7.
    w = np.array([[1.0, 2.0 ** -8, 2.0 ** -24, 2.0 ** -24], [0.5, 0.5, 0.0, 0.0]], dtype=np.float32)
    sr = np.array([[0, 1, 2, 3], [-1, -1, -1, -1]], dtype=np.int32)
    y = moe.combine(eo, sr, w, 2, H)
    assert np.all(y[0] == 0x3F80)
    assert np.all(y[1] == 0)
