"""Pins of the oracle's FP8 dequantisation, x = bf16(fp32(code) * scale).

The NCCL EP page ("NCCL EP架构解析", section 2.1) sends the FP8 payload with a scale tensor; the
expert FFN here consumes bf16, so each packed FP8 row is turned back into bf16 before the GEMM:
the e4m3 code's value times its block's fp32 scale, as one fp32 product, then rounded to bf16
(nearest, ties to even).  Each hand-derived case below changes its result if either rounding step is
dropped or done in another precision; the last test checks the same composition against torch's own
e4m3 -> fp32 conversion, fp32 multiply and bf16 cast.
"""
import numpy as np
import torch

from oracle import moe

BF16_ONE = 0x3F80


def dq(code: int, scale: float) -> float:
    """The oracle's dequantised value of one code in a one-block row with this scale."""
    codes = np.full((1, moe.QBLOCK), code, dtype=np.uint8)
    scales = np.array([[scale]], dtype=np.float32)
    out = moe.dequantize_fp8_rows(codes, scales)
    assert out.shape == (1, moe.QBLOCK) and np.all(out == out[0, 0])
    return float(out[0, 0])


def bits_of(v: float) -> int:
    return int(np.array([v], dtype=np.float32).view(np.uint32)[0] >> 16)


def test_exact_product_on_a_bf16_midpoint_ties_to_even():
    # code 0x38 = 1.0; scale 1 + 2^-8 is exact in fp32 and the product 1.00390625 lies halfway
    # between the bf16 neighbours 1.0 (even fraction) and 1.0078125: ties to even give 1.0
    assert dq(0x38, 1.0 + 2.0 ** -8) == 1.0
    # scale 1 + 3 * 2^-8: halfway between 1.0078125 (odd) and 1.015625 (even) -> 1.015625
    assert dq(0x38, 1.0 + 3 * 2.0 ** -8) == 1.015625
    # just past the midpoint goes up
    assert dq(0x38, float(np.nextafter(np.float32(1.0 + 2.0 ** -8), np.float32(2)))) == 1.0078125


def test_fp32_product_rounding_decides_the_bf16_value():
    # code 0x3D = 1 + 5/8 = 1.625 and scale = 0x1.3c4ec6p-1 (an fp32 value).  The exact product is
    # 1 + 2^-8 + 5.2e-8: above the bf16 midpoint 1 + 2^-8, so rounding it once would give 1.0078125.
    # The fp32 product rounds it to the midpoint itself (5.2e-8 < 2^-24, half an fp32 ulp in
    # [1, 2)), and the bf16 rounding of that tie goes to the even neighbour 1.0.
    scale = float.fromhex("0x1.3c4ec6p-1")
    assert np.float32(scale) == scale
    assert bits_of(dq(0x3D, scale)) == BF16_ONE
    assert bits_of(dq(0xBD, scale)) == 0x8000 | BF16_ONE      # sign bit of the code carries over


def test_subnormal_scales_and_products():
    # 2^-9 (code 0x01, smallest e4m3 subnormal) * 2^-130 = 2^-139: an fp32 subnormal, but below
    # half the smallest bf16 subnormal 2^-133, so the bf16 value is +0
    v = dq(0x01, 2.0 ** -130)
    assert v == 0.0 and not np.signbit(v)
    # 448 * 2^-140 = 3.5 * 2^-133: halfway between 3 and 4 bf16 subnormal quanta -> 4 * 2^-133
    assert dq(0x7E, 2.0 ** -140) == 2.0 ** -131
    # 2^-9 * 2^-149 underflows in the fp32 product itself
    assert dq(0x01, 2.0 ** -149) == 0.0
    # an exact product in the bf16 subnormal range stays as it is: 1.0 * 5 * 2^-133
    assert dq(0x38, 5 * 2.0 ** -133) == 5 * 2.0 ** -133


def test_zero_block_and_scale_one():
    # an all-zero block is sent with scale 1 and codes 0 (or 0x80 for -0): the values are +-0
    assert dq(0x00, 1.0) == 0.0
    v = dq(0x80, 1.0)
    assert v == 0.0 and np.signbit(v)
    # with scale 1 every finite code's value is exactly representable in bf16 (3-bit fraction)
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    rows = np.repeat(codes[:, None], moe.QBLOCK, axis=1)
    got = moe.dequantize_fp8_rows(rows, np.ones((codes.size, 1), dtype=np.float32))[:, 0]
    want = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(got, want)


def test_matches_torch_e4m3_to_fp32_times_scale_to_bf16():
    g = np.random.default_rng(8)
    n_rows, n_blocks = 600, 4
    codes = g.integers(0, 256, size=(n_rows, n_blocks * moe.QBLOCK), dtype=np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x3C                      # no NaN codes in a payload
    # scales as the quantiser makes them (amax / 448 for amax spread over many decades), plus
    # full-mantissa random values, subnormal ones and 1.0
    amax = np.exp(g.uniform(np.log(1e-30), np.log(1e4), size=(n_rows, n_blocks)))
    scales = (amax.astype(np.float32) / np.float32(448.0)).astype(np.float32)
    scales[::7] = g.uniform(0.5, 2.0, size=scales[::7].shape).astype(np.float32)
    scales[3::11] = (g.uniform(1, 2 ** 20, size=scales[3::11].shape) * 2.0 ** -149).astype(np.float32)
    scales[5::13] = 1.0
    got = moe.dequantize_fp8_rows(codes, scales)
    q = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float32)
    s = torch.from_numpy(scales).repeat_interleave(moe.QBLOCK, dim=1)
    ref = (q * s).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(np.signbit(got), np.signbit(ref))
    assert np.array_equal(got, ref)
