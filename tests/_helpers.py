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


def to_dev_bf16_from_bits(bits: np.ndarray, device) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)
