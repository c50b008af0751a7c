"""Pins of the oracle's bf16 and e4m3 rounding against the formats' definitions and torch's casts."""
import numpy as np
import torch

from oracle.numerics import (bf16_bits, bf16_from_bits, bf16_round, e4m3_decode,
                             e4m3_encode_satfinite, e4m3_value_table)


def test_e4m3_table_landmarks():
    v = e4m3_value_table()
    assert v[0x00] == 0.0 and np.signbit(v[0x80])
    assert v[0x01] == 2.0 ** -9            # smallest subnormal
    assert v[0x07] == 7 * 2.0 ** -9        # largest subnormal
    assert v[0x08] == 2.0 ** -6            # smallest normal
    assert v[0x38] == 1.0                  # exponent field 7 = bias
    assert v[0x7E] == 448.0 and v[0xFE] == -448.0
    assert np.isnan(v[0x7F]) and np.isnan(v[0xFF])
    assert np.count_nonzero(np.isnan(v)) == 2
    pos = v[:127]
    assert np.all(np.diff(pos) > 0)        # codes 0..126 are increasing
    assert np.array_equal(v[0x80:0xFF], -v[0:0x7F])


def test_e4m3_roundtrip_all_codes():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    back = e4m3_encode_satfinite(e4m3_decode(codes))
    assert np.array_equal(back, codes)


def test_e4m3_midpoints_tie_to_even():
    v = e4m3_value_table()[:127]
    for c in range(126):
        mid = (v[c] + v[c + 1]) / 2
        even = c if c % 2 == 0 else c + 1
        assert e4m3_encode_satfinite(mid) == even, c
        assert e4m3_encode_satfinite(np.nextafter(mid, 0)) == c
        assert e4m3_encode_satfinite(np.nextafter(mid, 1e9)) == c + 1
        assert e4m3_encode_satfinite(-mid) == (0x80 | even)


def test_e4m3_saturation_and_specials():
    assert e4m3_encode_satfinite(448.0) == 0x7E
    assert e4m3_encode_satfinite(464.0) == 0x7E      # would round past the top code: saturate
    assert e4m3_encode_satfinite(1e30) == 0x7E
    assert e4m3_encode_satfinite(np.inf) == 0x7E
    assert e4m3_encode_satfinite(-np.inf) == 0xFE
    assert e4m3_encode_satfinite(np.nan) == 0x7F
    assert e4m3_encode_satfinite(2.0 ** -10) == 0x00  # half the smallest subnormal: tie to even 0
    assert e4m3_encode_satfinite(-1e-30) == 0x80      # negative underflow keeps the sign


def test_e4m3_matches_torch_cast_in_range():
    g = np.random.default_rng(1)
    x = np.concatenate([g.normal(0, 50, 200000), g.uniform(-448, 448, 200000),
                        g.normal(0, 2.0 ** -7, 100000)]).astype(np.float32)
    ours = e4m3_encode_satfinite(x)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)


def test_bf16_matches_torch_cast():
    g = np.random.default_rng(2)
    bits = g.integers(0, 2 ** 32, 2_000_000, dtype=np.uint64).astype(np.uint32)
    x = bits.view(np.float32)
    x = x[np.isfinite(x)]
    ours = bf16_bits(x)
    ref = torch.from_numpy(x.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_bf16_midpoints_tie_to_even():
    hi = np.arange(0, 0x7F7F, dtype=np.uint32)
    lo_v = bf16_from_bits(hi.astype(np.uint16)).astype(np.float64)
    up_v = bf16_from_bits((hi + 1).astype(np.uint16)).astype(np.float64)
    mid = (lo_v + up_v) / 2
    got = bf16_bits(mid).astype(np.uint32)
    expect = np.where(hi % 2 == 0, hi, hi + 1)
    assert np.array_equal(got, expect)
    # just off the midpoint goes to the nearer neighbour
    assert np.array_equal(bf16_bits(np.nextafter(mid, 0)).astype(np.uint32)[1:], hi[1:])


def test_bf16_overflow_and_specials():
    big = bf16_from_bits(np.uint16(0x7F7F)).astype(np.float64)  # largest finite bf16
    ulp = 2.0 ** (127 - 7)
    assert bf16_round(big + ulp / 2 * 0.999)[()] == big
    assert np.isinf(bf16_round(big + ulp / 2)[()])             # tie to even -> 2^128 -> inf
    assert bf16_bits(np.nan) == 0x7FC0
    assert bf16_bits(-0.0) == 0x8000
    assert bf16_bits(2.0 ** -133) == 0x0001                    # smallest bf16 subnormal
    assert bf16_bits(2.0 ** -134) == 0x0000                    # tie to even -> 0
