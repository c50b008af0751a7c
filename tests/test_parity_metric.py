"""The element-wise parity bar used by the GPU tests flags what it should, on the CPU."""
import numpy as np

from _helpers import assert_close_bf16, bf16_values, parity_report
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


def test_combine_output_is_judged_against_the_size_of_its_summands():
    # y = 0.5 * a + 0.5 * b with a ~ -b: y is near zero, and a one-ulp difference in a (as two
    # fp32-accumulated FFNs may round differently) moves y by half an ulp of a
    from _helpers import combine_magnitude
    a = np.array([[1.5, 2.0]]), np.array([[-1.49, 1.0]])
    eo = bf16_bits(np.concatenate(a))
    sr = np.array([[0, 1]])
    w = np.array([[0.5, 0.5]], dtype=np.float32)
    ref = bf16_bits(0.5 * bf16_values(eo[0]) + 0.5 * bf16_values(eo[1]))[None, :]
    eo2 = eo.copy()
    eo2[0, 0] += 1                                   # one ulp of 1.5 = 2^-7
    got = bf16_bits(0.5 * bf16_values(eo2[0]) + 0.5 * bf16_values(eo2[1]))[None, :]
    assert parity_report(got, ref)["n_bad"] == 1     # judged against |y| ~ 0.004 alone: fails
    rep = parity_report(got, ref, combine_magnitude(eo, sr, w))
    assert rep["n_bad"] == 0                          # against 0.5*1.5 + 0.5*1.49: passes


def test_row_allowance_of_expert_out_covers_one_flipped_h_and_nothing_like_a_wrong_row():
    import torch
    from _helpers import ffn_row_atol
    g = np.random.default_rng(4)
    S, F, H = 6, 64, 32
    h = g.normal(size=(S, F))
    wd = g.normal(0, 0.05, size=(1, H, F))
    hb = bf16_bits(h)
    eo_ref = bf16_bits(bf16_values(hb) @ bf16_values(bf16_bits(wd[0])).T)
    atol = ffn_row_atol(hb, np.array([0, S]), torch.from_numpy(bf16_values(bf16_bits(wd))))
    # the largest h of row 2 rounded one ulp the other way
    h2 = hb.copy()
    f = int(np.argmax(np.abs(bf16_values(hb[2]))))
    h2[2, f] += 1
    eo_flip = bf16_bits(bf16_values(h2) @ bf16_values(bf16_bits(wd[0])).T)
    assert parity_report(eo_flip, eo_ref, row_atol=atol)["n_bad"] == 0
    # another row's output in row 2: far outside
    eo_bad = eo_ref.copy()
    eo_bad[2] = eo_ref[3]
    assert parity_report(eo_bad, eo_ref, row_atol=atol)["n_bad"] > H // 2
