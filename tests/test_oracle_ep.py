"""The expert-parallel pieces of the oracle against what fixes them independently.

* ``ep_segment_rows`` (the per-peer block layouts) against a sort-based restatement: a packed
  a-major layout is the rank of (a, b, q) in lexicographic order, a b-major one the rank of
  (b, a, q); with a block stride, the block's first row is block * stride and the rows inside the
  block follow the same order.
* ``ep_pipeline`` (each rank routes and dispatches its own tokens, per-destination blocks cross
  the ranks, every rank runs its own experts, the rows return and each rank combines its tokens)
  against the single-device ``pipeline`` over the rank-major concatenation of all ranks' tokens:
  the two orderings put the same operands in front of the same arithmetic, so the outputs are
  equal bit for bit (the NCCL EP page, sections 1 and 2: the exchange moves rows and changes no
  value).  A planted mistake in the exchange (a source block returned to the wrong sender) fails.
"""
import numpy as np
import pytest

import moe_inputs as mi
from oracle import moe
from oracle.numerics import bf16_bits


def _sorted_positions(counts, order, stride):
    c = np.asarray(counts)
    A, B = c.shape
    keys = [(a, b, q) for a in range(A) for b in range(B) for q in range(int(c[a, b]))]
    major = (lambda t: t[0]) if order == 0 else (lambda t: t[1])
    ordered = sorted(keys, key=(lambda t: t) if order == 0 else (lambda t: (t[1], t[0], t[2])))
    pos = {}
    if stride == 0:
        for i, key in enumerate(ordered):
            pos[key] = i
        return pos
    within = {}
    for key in ordered:
        m = major(key)
        pos[key] = m * stride + within.get(m, 0)
        within[m] = within.get(m, 0) + 1
    return pos


@pytest.mark.parametrize("order", [0, 1])
@pytest.mark.parametrize("padded", [False, True])
def test_segment_rows_match_a_sort(order, padded):
    rng = np.random.default_rng(7)
    for A, B in [(1, 1), (2, 3), (4, 2), (3, 5)]:
        counts = rng.integers(0, 5, size=(A, B))
        counts[rng.integers(0, A), :] = 0                     # an empty block
        blocks = counts.sum(axis=1) if order == 0 else counts.sum(axis=0)
        stride = int(blocks.max()) + 2 if padded else 0
        assert moe.ep_segment_rows(counts, order, stride) == _sorted_positions(counts, order,
                                                                                 stride)


def test_regroup_moves_rows_and_back():
    rng = np.random.default_rng(3)
    counts = rng.integers(0, 4, size=(3, 4))
    n = int(counts.sum())
    src = rng.integers(0, 1 << 16, size=(n, 5)).astype(np.uint16)
    grouped, off = moe.ep_regroup(counts, src, 0, 0, np.zeros_like(src), 1, 0)
    assert list(off) == [0] + list(np.cumsum(counts.sum(axis=0)))
    # expert-major: the rows of column b from every a, a ascending
    expect, base = [], np.concatenate([[0], np.cumsum(counts.sum(axis=1))])
    for b in range(4):
        for a in range(3):
            lo = base[a] + counts[a, :b].sum()
            expect.extend(src[lo:lo + counts[a, b]])
    assert np.array_equal(grouped, np.array(expect).reshape(n, 5))
    back, _ = moe.ep_regroup(counts, grouped, 1, 0, np.zeros_like(src), 0, 0)
    assert np.array_equal(back, src)
    # padded blocks of stride M and back
    M = int(counts.sum(axis=1).max())
    pad, _ = moe.ep_regroup(counts, src, 0, 0, np.zeros((3 * M, 5), np.uint16), 0, M)
    unpad, _ = moe.ep_regroup(counts, pad, 0, M, np.zeros_like(src), 0, 0)
    assert np.array_equal(unpad, src)


def _ep_case(name, R, seed=0):
    w = mi.get(name)
    d = mi.make_ep_inputs(w, R, seed)
    lg = [t.numpy() for t in d["logits"]]
    xs = [bf16_bits(t.float().numpy()) for t in d["x"]]
    wb = [bf16_bits(d[key].float().numpy()) for key in ("w_gate", "w_up", "w_down")]
    return w, lg, xs, wb


@pytest.mark.parametrize("R", [2, 4])
@pytest.mark.parametrize("fp8", [False, True])
def test_ep_pipeline_equals_single_device_on_concatenated_tokens(R, fp8):
    w, lg, xs, wb = _ep_case("tiny", R)
    # a shorter token count keeps the fp64 FFN quick; rank 1's tokens avoid rank 0's experts
    lg = [a[:48].copy() for a in lg]
    xs = [a[:48].copy() for a in xs]
    E_loc = w.E // R
    lg[1][:, :E_loc] -= 50.0
    ys = moe.ep_pipeline(lg, xs, *wb, w.k, fp8=fp8)
    ref = moe.pipeline(np.concatenate(lg), np.concatenate(xs), *wb, w.k, R, fp8=fp8)
    assert np.array_equal(np.concatenate(ys), ref["y"])


def test_ep_pipeline_with_an_idle_expert_rank_and_k_above_experts_per_rank():
    # E_loc = 2 < k = 3: a token can send up to 2 rows to one rank; rank 3's experts get no rows
    rng = np.random.default_rng(11)
    R, T, E, k, H, F = 4, 20, 8, 3, 128, 64
    lg = [rng.standard_normal((T, E)).astype(np.float32) for _ in range(R)]
    for a in lg:
        a[:, 6:] -= 100.0
    xs = [bf16_bits(rng.standard_normal((T, H))) for _ in range(R)]
    wb = [bf16_bits(rng.standard_normal(s) * 0.05) for s in [(E, F, H), (E, F, H), (E, H, F)]]
    ys = moe.ep_pipeline(lg, xs, *wb, k)
    ref = moe.pipeline(np.concatenate(lg), np.concatenate(xs), *wb, k, R)
    assert np.array_equal(np.concatenate(ys), ref["y"])


def test_planted_exchange_mistake_is_caught(monkeypatch):
    """Returning source 0's rows to source 1 (a swapped sender) breaks the invariant."""
    w, lg, xs, wb = _ep_case("tiny", 2)
    lg = [a[:32].copy() for a in lg]
    xs = [a[:32].copy() for a in xs]
    real = moe.ep_regroup

    def swapped(counts, src, so, ss, dst, do, ds):
        out, off = real(counts, src, so, ss, dst, do, ds)
        if so == 1 and do == 0:               # the return trip: reverse the source blocks
            c = np.asarray(counts)
            n0 = int(c[0].sum())
            out = np.concatenate([out[n0:], out[:n0]])
        return out, off

    monkeypatch.setattr(moe, "ep_regroup", swapped)
    ys = moe.ep_pipeline(lg, xs, *wb, w.k)
    ref = moe.pipeline(np.concatenate(lg), np.concatenate(xs), *wb, w.k, 2)
    assert not np.array_equal(np.concatenate(ys), ref["y"])
