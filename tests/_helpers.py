"""Test-only helpers: tensor <-> numpy bit views and error metrics."""
from __future__ import annotations

import numpy as np
import torch


def bits16(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> uint16 bit patterns (numpy, CPU)."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def bytes8(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().view(torch.uint8).numpy()


def np_(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().numpy()


def bf16_values(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def rel_max_err(got_bits, ref_bits) -> float:
    """max |got - ref| / max |ref| over bf16 arrays (the parity metric for FFN and combine outputs)."""
    g, r = bf16_values(got_bits), bf16_values(ref_bits)
    denom = np.max(np.abs(r))
    if denom == 0:
        return float(np.max(np.abs(g)))
    return float(np.max(np.abs(g - r)) / denom)


# Element-wise parity bar for bf16 outputs of the FFN and the whole path: an element fails when
# |got - ref| > RTOL * mag + ATOL_REL * max|ref|, where mag is the element's magnitude scale: |ref|
# itself, or for a sum whose inputs were rounded to bf16 (the combine's y = sum_j w_j eo_j) the
# magnitude of its summands, sum_j |w_j eo_j|, since a one-ulp difference in an input moves the sum
# by that much however far the terms cancel.  RTOL covers one bf16 rounding step (2^-8 of the value)
# with margin; the absolute term, scaled to the tensor's magnitude, covers elements near zero where
# fp32-accumulated dot products cancel (their error is set by the size of the summands).
RTOL = 1e-2
ATOL_REL = 1e-3


def combine_magnitude(expert_out_bits, slot_row, topk_w) -> np.ndarray:
    """sum_j |w[t,j]| |expert_out[slot_row[t,j]]| per output element (float64, [T, H])."""
    eo = np.abs(bf16_values(expert_out_bits))
    sr = np.asarray(slot_row, dtype=np.int64)
    w = np.abs(np.asarray(topk_w, dtype=np.float64))
    mag = np.zeros((sr.shape[0], eo.shape[1] if eo.ndim == 2 else 0))
    for j in range(sr.shape[1]):
        ok = sr[:, j] >= 0
        if np.any(ok):
            mag[ok] += w[ok, j][:, None] * eo[sr[ok, j]]
    return mag


# A one-ulp difference in an h value (the two sides accumulate gate and up in fp32 and fp64, so a
# value near a bf16 rounding boundary can round either way) moves an output of the second GEMM by at
# most ulp(h) * |w| <= 2^-8 |h| |w|.  The row allowance of expert_out is four such flips of the row's
# largest |h| against the expert's largest |w_down|; a wrong tile, row or expert errs by the size of
# the output itself, far above it.
FLIPS_PER_ROW = 4


def ffn_row_atol(h_bits, expert_offsets, w_down) -> np.ndarray:
    """Per packed row: FLIPS_PER_ROW * 2^-8 * max_f |h[r, f]| * max |W_down[expert of r]|."""
    h = np.abs(bf16_values(h_bits))
    S = h.shape[0]
    if S == 0:
        return np.zeros(0)
    off = np.asarray(expert_offsets, dtype=np.int64)
    wd = w_down.detach().abs().float().reshape(w_down.shape[0], -1).amax(dim=1).cpu().numpy()
    expert = np.searchsorted(off, np.arange(S), side="right") - 1
    return FLIPS_PER_ROW * 2.0 ** -8 * h.max(axis=1) * wd[expert].astype(np.float64)


def combine_row_atol(expert_out_ref_bits, slot_row, topk_w, eo_row_atol) -> np.ndarray:
    """Per token: the expert_out allowance of its kept slots carried through the combine weights,
    sum_j |w_j| (ATOL_REL max|expert_out| + eo_row_atol[row_j])."""
    eo_scale = float(np.max(np.abs(bf16_values(expert_out_ref_bits)))) if np.size(expert_out_ref_bits) else 0.0
    sr = np.asarray(slot_row, dtype=np.int64)
    w = np.abs(np.asarray(topk_w, dtype=np.float64))
    out = np.zeros(sr.shape[0])
    for j in range(sr.shape[1]):
        ok = sr[:, j] >= 0
        out[ok] += w[ok, j] * (ATOL_REL * eo_scale + eo_row_atol[sr[ok, j]])
    return out


def parity_report(got_bits, ref_bits, mag=None, row_atol=None) -> dict:
    """max |got - ref| / max |ref|, the Frobenius relative error, and the count of elements outside
    the element-wise bar (NaN on either side counts as outside).  ``row_atol``: an extra absolute
    allowance per row."""
    g, r = bf16_values(got_bits), bf16_values(ref_bits)
    assert g.shape == r.shape, (g.shape, r.shape)
    if g.size == 0:
        return {"rel_max": 0.0, "frob": 0.0, "n_bad": 0, "n": 0}
    d = np.abs(g - r)
    scale = float(np.max(np.abs(r)))
    m = np.abs(r) if mag is None else np.maximum(np.asarray(mag, dtype=np.float64), np.abs(r))
    bound = RTOL * m + ATOL_REL * scale
    if row_atol is not None:
        bound = bound + np.asarray(row_atol, dtype=np.float64).reshape(-1, *([1] * (g.ndim - 1)))
    bad = ~(d <= bound)                      # NaN compares false: counted as bad
    nr = float(np.linalg.norm(r))
    rep = {"rel_max": float(np.max(d) / scale) if scale > 0 else float(np.max(d)),
           "frob": float(np.linalg.norm(np.nan_to_num(g - r, nan=np.inf)) / nr) if nr > 0 else 0.0,
           "n_bad": int(np.count_nonzero(bad)), "n": int(g.size)}
    if rep["n_bad"]:
        # the worst elements relative to their bound: index, got, ref, bound, magnitude scale
        ratio = np.where(bad, np.nan_to_num(d / np.maximum(bound, 1e-300), nan=np.inf), 0.0)
        worst = np.argsort(ratio.ravel())[::-1][:6]
        rep["worst"] = [(tuple(int(i) for i in np.unravel_index(f, g.shape)), float(g.flat[f]),
                         float(r.flat[f]), float(bound.flat[f]), float(m.flat[f])) for f in worst
                        if bad.flat[f]]
        rep["max_abs_ref"] = scale
    return rep


def assert_close_bf16(got_bits, ref_bits, what: str = "", mag=None, row_atol=None) -> dict:
    """The parity bar for a bf16 output tensor: max-relative error <= RTOL and no element outside
    the element-wise bar (``mag``: the elements' magnitude scale, default |ref|; ``row_atol``: an
    extra absolute allowance per row)."""
    rep = parity_report(got_bits, ref_bits, mag, row_atol)
    assert rep["rel_max"] <= RTOL and rep["n_bad"] == 0, f"{what}: {rep}"
    return rep


def to_dev_bf16_from_bits(bits: np.ndarray, device) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def assert_ffn_and_combine(h_got, eo_got, y_got, h_ref, eo_ref, y_ref, expert_offsets, w_down,
                           slot_row, topk_w, what: str = ""):
    """The parity bar for h, expert_out (with the h-flip row allowance) and y (with the expert_out
    allowance carried through the combine, and the size of its summands as magnitude)."""
    assert_close_bf16(h_got, h_ref, f"{what} h")
    eo_atol = ffn_row_atol(h_ref, expert_offsets, w_down)
    assert_close_bf16(eo_got, eo_ref, f"{what} expert_out", row_atol=eo_atol)
    if y_got is not None:
        assert_close_bf16(y_got, y_ref, f"{what} y", combine_magnitude(eo_ref, slot_row, topk_w),
                          combine_row_atol(eo_ref, slot_row, topk_w, eo_atol))
