"""The oracle's backward pass against what fixes it independently.

* Finite differences: an fp64 forward written here from the definitions (top-k weights from the
  logits, the kept slots of the plan, SwiGLU experts, the weighted sum), central differences of
  L = sum(y * dy) with respect to the token activations, the three weight tensors and the router
  logits must equal the oracle's exact gradients (``exact=True``: no bf16 rounding), with
  renormalised and full-softmax weights and with a capacity that drops slots.  The selection is
  piecewise constant, so the logits are drawn with gaps far above the difference step.
* The rounded gradients (bf16 at the stated boundaries) stay within the bf16 error of the exact
  ones.
* A planted mistake (the SwiGLU derivative without its (1 + g (1 - s)) factor) fails.
"""
import numpy as np
import pytest

from oracle import moe
from oracle.numerics import bf16_bits, bf16_from_bits


def _case(seed, T=6, H=8, F=6, E=4, k=2, scale=0.4):
    rng = np.random.default_rng(seed)
    # logits on a coarse grid with distinct values per token: selection never flips within eps
    logits = np.stack([rng.permutation(E).astype(np.float64) * 0.7 + rng.normal(0, 0.05, E)
                       for _ in range(T)]).astype(np.float32)
    xb = bf16_bits(rng.normal(0, 1, (T, H)))
    wg = bf16_bits(rng.normal(0, scale, (E, F, H)))
    wu = bf16_bits(rng.normal(0, scale, (E, F, H)))
    wd = bf16_bits(rng.normal(0, scale, (E, H, F)))
    dyb = bf16_bits(rng.normal(0, 1, (T, H)))
    return logits, xb, wg, wu, wd, dyb, k


def fwd64(logits, x, wg, wu, wd, idx, slot_row, renormalize):
    """y = sum over kept slots of w_j * (silu(x Wg_e^T) * (x Wu_e^T)) Wd_e^T, all fp64."""
    T, E = logits.shape
    y = np.zeros((T, x.shape[1]))
    for t in range(T):
        l = logits[t].astype(np.float64)
        if renormalize:
            sel = l[idx[t]]
            ex = np.exp(sel - sel.max())
            wt = ex / ex.sum()
        else:
            ex = np.exp(l - l.max())
            wt = (ex / ex.sum())[idx[t]]
        for j, e in enumerate(idx[t]):
            if slot_row[t, j] < 0:
                continue
            g = wg[e] @ x[t]
            u = wu[e] @ x[t]
            h = g / (1 + np.exp(-g)) * u
            y[t] += wt[j] * (wd[e] @ h)
    return y


def _grads_fd(logits, x, wg, wu, wd, dy, idx, slot_row, renormalize, eps=1e-6):
    def L(lg=logits, xx=x, g=wg, u=wu, d=wd):
        return float(np.sum(fwd64(lg, xx, g, u, d, idx, slot_row, renormalize) * dy))

    def fd(arr, name):
        out = np.zeros_like(arr, dtype=np.float64)
        it = np.nditer(arr, flags=["multi_index"])
        for _ in it:
            i = it.multi_index
            a = arr.astype(np.float64).copy()
            a[i] += eps
            plus = L(**{name: a})
            a[i] -= 2 * eps
            minus = L(**{name: a})
            out[i] = (plus - minus) / (2 * eps)
        return out

    return {"dx": fd(x, "xx"), "d_w_gate": fd(wg, "g"), "d_w_up": fd(wu, "u"),
            "d_w_down": fd(wd, "d"), "d_logits": fd(logits.astype(np.float64), "lg")}


@pytest.mark.parametrize("renormalize,cf", [(True, 0.0), (False, 0.0), (True, 0.75)])
def test_exact_backward_equals_finite_differences(renormalize, cf):
    logits, xb, wg, wu, wd, dyb, k = _case(1 + int(renormalize) + int(cf * 4))
    T, E = logits.shape
    R = 2
    fwd = moe.pipeline(logits, xb, wg, wu, wd, k, R, cf, renormalize=renormalize)
    if cf:
        assert (fwd["slot_row"] < 0).any()      # the capacity drops some slots
    g = moe.backward(fwd, dyb, logits, wg, wu, wd, renormalize=renormalize, exact=True)
    vals = [bf16_from_bits(a).astype(np.float64) for a in (xb, wg, wu, wd, dyb)]
    fd = _grads_fd(logits.astype(np.float64), vals[0], vals[1], vals[2], vals[3], vals[4],
                   fwd["topk_idx"], fwd["slot_row"], renormalize)
    for name in ("dx", "d_w_gate", "d_w_up", "d_w_down", "d_logits"):
        got = np.asarray(g[name], dtype=np.float64)
        ref = fd[name]
        scale = max(np.max(np.abs(ref)), 1e-3)
        assert np.max(np.abs(got - ref)) <= 1e-6 * scale + 1e-8, name


def test_rounded_backward_is_close_to_exact():
    logits, xb, wg, wu, wd, dyb, k = _case(7, T=12, H=16, F=8, E=4)
    fwd = moe.pipeline(logits, xb, wg, wu, wd, k, 2)
    a = moe.backward(fwd, dyb, logits, wg, wu, wd)
    b = moe.backward(fwd, dyb, logits, wg, wu, wd, exact=True)
    ra = bf16_from_bits(a["dx"]).astype(np.float64)
    assert np.max(np.abs(ra - b["dx"])) <= 0.03 * np.max(np.abs(b["dx"]))
    for name in ("d_w_gate", "d_w_up", "d_w_down", "d_logits"):
        x, y = np.asarray(a[name], np.float64), np.asarray(b[name], np.float64)
        assert np.max(np.abs(x - y)) <= 0.03 * np.max(np.abs(y)), name


def test_planted_swiglu_derivative_mistake_is_caught(monkeypatch):
    """silu'(g) = s (1 + g (1 - s)): the oracle's expert backward with the bracket dropped (planted
    in a copy of its source) no longer matches the finite differences."""
    import inspect
    logits, xb, wg, wu, wd, dyb, k = _case(3)
    fwd = moe.pipeline(logits, xb, wg, wu, wd, k, 2)
    vals = [bf16_from_bits(a).astype(np.float64) for a in (xb, wg, wu, wd, dyb)]
    fd = _grads_fd(logits.astype(np.float64), vals[0], vals[1], vals[2], vals[3], vals[4],
                   fwd["topk_idx"], fwd["slot_row"], True)
    good = moe.backward(fwd, dyb, logits, wg, wu, wd, exact=True)
    assert np.allclose(good["d_w_gate"], fd["d_w_gate"], atol=1e-6)
    text = inspect.getsource(moe.expert_backward)
    assert "(1.0 + g * (1.0 - sg))" in text
    ns = dict(vars(moe))
    exec(compile(text.replace("(1.0 + g * (1.0 - sg))", "1.0"), "planted", "exec"), ns)
    monkeypatch.setattr(moe, "expert_backward", ns["expert_backward"])
    bad = moe.backward(fwd, dyb, logits, wg, wu, wd, exact=True)
    assert not np.allclose(bad["d_w_gate"], fd["d_w_gate"], atol=1e-4)
