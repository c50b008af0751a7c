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


def parity_report(got_bits, ref_bits, mag=None) -> dict:
    """max |got - ref| / max |ref|, the Frobenius relative error, and the count of elements outside
    the element-wise bar (NaN on either side counts as outside)."""
    g, r = bf16_values(got_bits), bf16_values(ref_bits)
    assert g.shape == r.shape, (g.shape, r.shape)
    if g.size == 0:
        return {"rel_max": 0.0, "frob": 0.0, "n_bad": 0, "n": 0}
    d = np.abs(g - r)
    scale = float(np.max(np.abs(r)))
    m = np.abs(r) if mag is None else np.maximum(np.asarray(mag, dtype=np.float64), np.abs(r))
    bound = RTOL * m + ATOL_REL * scale
    bad = ~(d <= bound)                      # NaN compares false: counted as bad
    nr = float(np.linalg.norm(r))
    return {"rel_max": float(np.max(d) / scale) if scale > 0 else float(np.max(d)),
            "frob": float(np.linalg.norm(np.nan_to_num(g - r, nan=np.inf)) / nr) if nr > 0 else 0.0,
            "n_bad": int(np.count_nonzero(bad)), "n": int(g.size)}


def assert_close_bf16(got_bits, ref_bits, what: str = "", mag=None) -> dict:
    """The parity bar for a bf16 output tensor: max-relative error <= RTOL and no element outside
    the element-wise bar (``mag``: the elements' magnitude scale, default |ref|)."""
    rep = parity_report(got_bits, ref_bits, mag)
    assert rep["rel_max"] <= RTOL and rep["n_bad"] == 0, f"{what}: {rep}"
    return rep


def to_dev_bf16_from_bits(bits: np.ndarray, device) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)
