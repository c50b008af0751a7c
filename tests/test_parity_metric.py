"""The element-wise parity bar used by the GPU tests flags what it should, on the CPU."""
import numpy as np

from _helpers import assert_close_bf16, parity_report
from oracle.numerics import bf16_bits


def test_one_ulp_everywhere_passes():
    g = np.random.default_rng(0)
    ref = bf16_bits(g.normal(size=(64, 256)))
    got = (ref.astype(np.int32) + g.integers(-1, 2, size=ref.shape)).astype(np.uint16)
    got[ref & 0x7FFF == 0] = ref[ref & 0x7FFF == 0]           # no sign flips through zero
    rep = assert_close_bf16(got, ref)
    assert rep["n"] == ref.size and rep["rel_max"] < 1e-2


def test_a_small_element_far_off_fails_although_the_max_error_is_small():
    g = np.random.default_rng(1)
    v = g.normal(size=(32, 128))
    v[3, 7] = 0.01                       # an element far below the tensor's maximum (~4)
    ref = bf16_bits(v)
    w = v.copy()
    w[3, 7] = 0.02                       # 100% off, but only 0.01 absolute: rel_max about 2.5e-3
    rep = parity_report(bf16_bits(w), ref)
    assert rep["rel_max"] < 1e-2 and rep["n_bad"] == 1


def test_nan_counts_as_outside_the_bar():
    ref = bf16_bits(np.ones((4, 8)))
    got = ref.copy()
    got[1, 1] = 0x7FC0
    assert parity_report(got, ref)["n_bad"] == 1
