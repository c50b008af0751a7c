"""Pins of the oracle's FP8-weight FFN (W8A8 first projection) and its per-row FP8 quantiser.

FP8 and NVFP4 expert weights with block scales are what the DWDP page's NvFp4WeightView carries
("DWDP: 在NVL72上的高性能分布式权重数据并行", 关键优化实施).  Here the gate and up weights are e4m3
with one fp32 scale per output row, and each FFN input row is quantised on its own the same way,
so the first projection is sx * sw * sum(qx * qw); the down projection stays bf16."""
import math

import numpy as np
import pytest
import torch

from oracle import moe
from oracle.numerics import bf16_bits, bf16_from_bits, bf16_round, e4m3_value_table

E4M3 = e4m3_value_table()


def test_quantize_rows_hand_cases():
    q, s = moe.quantize_rows_fp8(np.array([[1.0, -2.0, 1344.0], [0.0, -0.0, 0.0]]))
    # row 0: amax 1344 -> scale 3; 1/3 -> 0.34375 (0x2B), -2/3 -> -0.6875 (0xB3), 448 -> 0x7E
    assert s.tolist() == [3.0, 1.0]
    assert q[0].tolist() == [0x2B, 0xB3, 0x7E]
    assert q[1].tolist() == [0x00, 0x80, 0x00]          # zero row: scale 1, codes keep the sign
    assert E4M3[0x2B] == 0.34375 and E4M3[0xB3] == -0.6875


def test_quantize_rows_largest_entry_maps_to_448_and_matches_torch():
    g = np.random.default_rng(5)
    x = (g.normal(size=(300, 512)) * np.exp(g.uniform(-20, 20, size=(300, 1)))).astype(np.float32)
    q, s = moe.quantize_rows_fp8(x)
    big = np.argmax(np.abs(x), axis=1)
    assert np.all((q[np.arange(300), big] & 0x7F) == 0x7E)
    ref = (torch.from_numpy(x) / torch.from_numpy(s)[:, None]).to(torch.float8_e4m3fn)
    assert np.array_equal(q, ref.view(torch.uint8).numpy())
    assert np.allclose(s, np.max(np.abs(x), axis=1) / np.float32(448), rtol=0, atol=0)


def exact_rows(g, rows, cols, pow2):
    """Rows of e4m3 values times a power of two, each row holding +-448 once: quantisation is exact
    (scale = the power of two) and the values are bf16 values too."""
    v = E4M3[g.integers(0, 126, size=(rows, cols))] * g.choice([-1.0, 1.0], size=(rows, cols))
    v[np.arange(rows), g.integers(0, cols, size=rows)] = 448.0
    return v * (2.0 ** np.asarray(pow2, dtype=np.float64))[:, None]


def test_w8_ffn_equals_bf16_ffn_when_quantisation_is_exact():
    g = np.random.default_rng(6)
    E, F, H, S = 3, 16, 64, 11
    off = np.array([0, 4, 4, 11])
    x = exact_rows(g, S, H, g.integers(-14, -6, size=S))
    wg = exact_rows(g, E * F, H, g.integers(-16, -10, size=E * F)).reshape(E, F, H)
    wu = exact_rows(g, E * F, H, g.integers(-16, -10, size=E * F)).reshape(E, F, H)
    wd = bf16_bits(g.normal(0, 0.1, size=(E, H, F)))
    qg, sg = zip(*[moe.quantize_rows_fp8(wg[e]) for e in range(E)])
    qu, su = zip(*[moe.quantize_rows_fp8(wu[e]) for e in range(E)])
    assert not np.all(np.array(sg) == 1.0)          # the scales take part
    h8, y8 = moe.expert_ffn_w8(x, off, np.stack(qg), np.stack(sg), np.stack(qu), np.stack(su), wd)
    h16, y16 = moe.expert_ffn(x, off, bf16_bits(wg), bf16_bits(wu), wd)
    assert np.array_equal(h8, h16) and np.array_equal(y8, y16)


def restated_w8(x, off, wg, wu, wd_bits):
    """Loops: per-row quantisation with Python floats (the fp64 quotient rounded once to fp32 is the
    IEEE fp32 quotient) and torch's e4m3 cast, then dot products in Python floats."""
    S, H = x.shape
    E, F, _ = wg.shape

    def qrow(row):
        amax = max(abs(float(v)) for v in row)
        sc = 1.0 if amax == 0 else float(np.float32(amax / 448.0))
        q = torch.tensor([float(np.float32(float(v) / sc)) for v in row],
                         dtype=torch.float32).to(torch.float8_e4m3fn).to(torch.float64).tolist()
        return [sc * c for c in q]

    h_all, y_all = [], []
    for r in range(S):
        e = int(np.searchsorted(off, r, side="right") - 1)
        xq = qrow(x[r])
        hrow = []
        for f in range(F):
            gq, uq = qrow(wg[e, f]), qrow(wu[e, f])
            gv = sum(a * b for a, b in zip(xq, gq))
            uv = sum(a * b for a, b in zip(xq, uq))
            hrow.append(float(bf16_round(gv / (1 + math.exp(-gv)) * uv)))
        wd = bf16_from_bits(wd_bits[e]).astype(np.float64)
        y_all.append([float(bf16_round(sum(hv * wd[o, f] for f, hv in enumerate(hrow))))
                      for o in range(H)])
        h_all.append(hrow)
    return np.array(h_all), np.array(y_all)


@pytest.mark.parametrize("seed", [0, 1])
def test_w8_ffn_matches_restatement_on_tiny_inputs(seed):
    g = np.random.default_rng(40 + seed)
    E, F, H, S = 2, 4, 32, 5
    off = np.array([0, 2, 5])
    x = bf16_from_bits(bf16_bits(g.normal(size=(S, H)))).astype(np.float64)
    wg = bf16_from_bits(bf16_bits(g.normal(0, 0.2, size=(E, F, H)))).astype(np.float64)
    wu = bf16_from_bits(bf16_bits(g.normal(0, 0.2, size=(E, F, H)))).astype(np.float64)
    wd = bf16_bits(g.normal(0, 0.2, size=(E, H, F)))
    qg, sg = zip(*[moe.quantize_rows_fp8(wg[e]) for e in range(E)])
    qu, su = zip(*[moe.quantize_rows_fp8(wu[e]) for e in range(E)])
    h8, y8 = moe.expert_ffn_w8(x, off, np.stack(qg), np.stack(sg), np.stack(qu), np.stack(su), wd)
    h_ref, y_ref = restated_w8(x, off, wg, wu, wd)
    hv = bf16_from_bits(h8).astype(np.float64)
    yv = bf16_from_bits(y8).astype(np.float64)
    # sums in another order may round a bf16 tie the other way: at most one ulp apart
    assert np.all(np.abs(hv - h_ref) <= 2.0 ** -7 * np.abs(h_ref) + 1e-30)
    assert np.all(np.abs(yv - y_ref) <= 2.0 ** -7 * np.abs(y_ref) + 2.0 ** -7 * np.max(np.abs(y_ref)) * 1e-2)
    # and the quantisation is not a no-op here: the bf16 FFN differs
    h16, _ = moe.expert_ffn(x, off, bf16_bits(wg), bf16_bits(wu), wd)
    assert not np.array_equal(h8, h16)
