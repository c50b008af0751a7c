"""Pins of the oracle router: brute-force sort, tie rule, distinct ids, softmax identities."""
import itertools
import math

import numpy as np
import pytest
from scipy.special import softmax

from oracle import moe


def brute_topk(row, k):
    keyed = sorted(range(len(row)), key=lambda e: (math.isnan(row[e]),
                                                   0.0 if math.isnan(row[e]) else -row[e], e))
    return keyed[:k]


@pytest.mark.parametrize("E,k", [(4, 1), (4, 2), (5, 3), (8, 8), (16, 4)])
def test_topk_equals_brute_force_sort(E, k):
    g = np.random.default_rng(E * 10 + k)
    l = g.normal(size=(50, E)).astype(np.float32)
    idx, w, routed = moe.route(l, k)
    for t in range(50):
        assert list(idx[t]) == brute_topk([float(v) for v in l[t]], k)
    assert routed.sum() == 50 * k


def test_ties_go_to_lower_expert_id():
    # integer logits make exact ties: every permutation of a row with repeated values
    base = [2.0, 2.0, 1.0, 1.0, 0.0]
    for perm in set(itertools.permutations(base)):
        row = np.array([perm], dtype=np.float32)
        idx, _, _ = moe.route(row, 3)
        twos = [e for e, v in enumerate(perm) if v == 2.0]
        ones = [e for e, v in enumerate(perm) if v == 1.0]
        assert list(idx[0]) == twos + ones[:1]


def test_ids_distinct_and_counts_sum():
    g = np.random.default_rng(3)
    l = g.normal(size=(300, 32)).astype(np.float32)
    idx, w, routed = moe.route(l, 6)
    assert all(len(set(r)) == 6 for r in idx)          # the heat map's zero diagonal
    assert routed.sum() == 300 * 6
    assert np.array_equal(routed, np.bincount(idx.ravel(), minlength=32))


def test_weights_renormalised_sum_to_one_and_descend():
    g = np.random.default_rng(4)
    l = g.normal(size=(200, 16)).astype(np.float32)
    _, w, _ = moe.route(l, 4)
    assert np.allclose(w.sum(1), 1.0, atol=1e-6)
    assert np.all(np.diff(w, axis=1) <= 0)


def test_k1_weight_is_one_and_kE_is_full_softmax():
    g = np.random.default_rng(5)
    l = g.normal(size=(64, 8)).astype(np.float32)
    _, w1, _ = moe.route(l, 1)
    assert np.all(w1 == 1.0)
    idx, w, _ = moe.route(l, 8)
    ref = softmax(l.astype(np.float64), axis=1)
    assert np.allclose(w, np.take_along_axis(ref, idx.astype(np.int64), 1), rtol=1e-6, atol=0)


def test_full_softmax_mode():
    g = np.random.default_rng(6)
    l = g.normal(size=(64, 16)).astype(np.float32)
    idx, w, _ = moe.route(l, 3, renormalize=False)
    ref = softmax(l.astype(np.float64), axis=1)
    assert np.allclose(w, np.take_along_axis(ref, idx.astype(np.int64), 1), rtol=1e-6, atol=0)
    assert np.all(w.sum(1) < 1.0)


def test_nonfinite_logits():
    nan, inf = np.nan, np.inf
    l = np.array([[nan, -inf, 1.0, 1.0],       # NaN ranks below -inf
                  [-inf, -inf, -inf, -inf],     # all -inf: equal weights
                  [0.0, inf, 5.0, inf],         # two +inf share the mass
                  [nan, nan, nan, 2.0]], dtype=np.float32)
    idx, w, _ = moe.route(l, 3)
    assert list(idx[0]) == [2, 3, 1]
    assert np.allclose(w[0], [0.5, 0.5, 0.0])
    assert list(idx[1]) == [0, 1, 2]
    assert np.allclose(w[1], [1 / 3] * 3)
    assert list(idx[2]) == [1, 3, 2]
    assert np.allclose(w[2], [0.5, 0.5, 0.0])
    assert list(idx[3]) == [3, 0, 1]
    assert np.allclose(w[3], [1.0, 0.0, 0.0])
