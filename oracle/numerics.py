"""Rounding to bf16 and to FP8 e4m3, written from the number formats' definitions.

TEST INFRASTRUCTURE ONLY.  Nothing under ``oracle/`` is part of the product path: only ``tests/``,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py``
may import it.  It shares no code with the CUDA library.

bf16: 1 sign bit, 8 exponent bits (bias 127, same range as IEEE binary32), 7 stored fraction bits,
so 8 significant bits.  Rounding is to nearest, ties to even; overflow past the largest finite
value (after rounding) gives infinity; NaN stays NaN.

e4m3 (OCP 8-bit floating point, "E4M3"): 1 sign bit, 4 exponent bits with bias 7, 3 fraction bits.
Exponent field 0 encodes subnormals m/8 * 2^-6; fields 1..15 encode (1 + m/8) * 2^(e-7), except
exponent 15 with fraction 7 (codes 0x7F / 0xFF), which is NaN.  There are no infinities; the
largest finite magnitude is 1.75 * 2^8 = 448.  The conversion used by the payload quantiser is
round to nearest, ties to even, saturating: finite values beyond 448 in magnitude become +-448.
"""
from __future__ import annotations

import numpy as np

__all__ = ["bf16_round", "bf16_bits", "bf16_from_bits", "e4m3_value_table", "e4m3_decode",
           "e4m3_encode_satfinite", "E4M3_MAX"]

E4M3_MAX = 448.0
_BF16_MIN_EXP = -126      # exponent of the smallest normal (shared with binary32)
_BF16_FRAC_BITS = 7


def bf16_round(v) -> np.ndarray:
    """Round float values (any float dtype, computed in fp64) to the nearest bf16 value, ties to
    even.  Returns float64 values that are exactly representable in bf16."""
    v = np.asarray(v, dtype=np.float64)
    out = np.empty_like(v)
    nan = np.isnan(v)
    inf = np.isinf(v)
    fin = ~(nan | inf)
    x = v[fin]
    # x = m * 2**ex with 0.5 <= |m| < 1, so the leading bit has weight 2**(ex-1).
    _, ex = np.frexp(x)
    lead = np.maximum(ex - 1, _BF16_MIN_EXP)          # subnormals share the quantum of 2**-126
    quantum = np.ldexp(1.0, lead - _BF16_FRAC_BITS)
    r = np.rint(x / quantum) * quantum                 # x/quantum is exact in fp64; rint: ties even
    r = np.where(np.abs(r) >= 2.0 ** 128, np.copysign(np.inf, x), r)
    r = np.where(x == 0, x, r)                         # keep the sign of zero
    out[fin] = r
    out[nan] = np.nan
    out[inf] = v[inf]
    return out


def bf16_bits(v) -> np.ndarray:
    """bf16 bit patterns (uint16) of ``bf16_round(v)``; NaN maps to the canonical 0x7FC0."""
    r = bf16_round(v)
    bits = (r.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    return np.where(np.isnan(r), np.uint16(0x7FC0), bits)


def bf16_from_bits(bits) -> np.ndarray:
    """float32 values of bf16 bit patterns (exact)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32)


def e4m3_value_table() -> np.ndarray:
    """Values of the 256 e4m3 codes (float64; NaN for 0x7F and 0xFF)."""
    vals = np.empty(256, dtype=np.float64)
    for code in range(256):
        sign = -1.0 if code & 0x80 else 1.0
        e = (code >> 3) & 0xF
        m = code & 0x7
        if e == 0xF and m == 0x7:
            vals[code] = np.nan
        elif e == 0:
            vals[code] = sign * (m / 8.0) * 2.0 ** -6
        else:
            vals[code] = sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return vals


_E4M3 = e4m3_value_table()
_POS = _E4M3[:127]            # codes 0x00..0x7E: 0, subnormals, normals up to 448, increasing


def e4m3_decode(codes) -> np.ndarray:
    return _E4M3[np.asarray(codes, dtype=np.uint8)]


def e4m3_encode_satfinite(v) -> np.ndarray:
    """Nearest e4m3 code (ties to the even code), saturating finite overflow to +-448.

    NaN maps to 0x7F.  The sign bit follows the sign of the input, so a negative value that
    rounds to zero gives 0x80."""
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    hi = np.searchsorted(_POS, a, side="left")          # first code with value >= a
    hi = np.clip(hi, 0, 126)
    lo = np.clip(hi - 1, 0, 126)
    d_lo = a - _POS[lo]
    d_hi = _POS[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo)
    code = np.where(a >= E4M3_MAX, 126, code)           # saturate (includes +-inf)
    code = code.astype(np.uint8)
    neg = np.signbit(v)
    code = np.where(neg, code | np.uint8(0x80), code).astype(np.uint8)
    return np.where(np.isnan(v), np.uint8(0x7F), code).astype(np.uint8)
