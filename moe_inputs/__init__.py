"""Seeded synthetic inputs for the MoE token shuffle (route -> dispatch -> SwiGLU FFN -> combine).

This module is shared by the CPU oracle, the CUDA path's tests and the benchmark.  It only draws
random numbers and shapes them; it holds none of the method's arithmetic (no top-k, no softmax, no
packing, no rounding rule other than torch's own cast of the drawn normals to bf16).

Workloads follow the five layer shapes the pages discuss:

* ``tiny``        T=128   H=256  E=8   k=2 R=4  F=512   (smallest case, oracle runs in full)
* ``decode``      T=128   H=4096 E=8   k=2 R=8  F=14336 (decode-style low latency, Mixtral-like
                  shape; NCCL-EP page, low-latency mode at 128 tokens)
* ``train``       T=4096  H=4096 E=8   k=2 R=8  F=14336 (training batch, per-expert logit bias
                  N(0, 0.5); NCCL-EP page, high-throughput mode at 4096 tokens)
* ``finegrained`` T=4096  H=7168 E=256 k=8 R=32 F=2048  (FP8 e4m3 payload with one fp32 scale per
                  128-element block; log-Zipf(1.2) expert bias)
* ``skewed``      T=16384 H=7168 E=128 k=2 R=16 F=2048  (capacity factor 1.25, drop in token order;
                  +3.0 logit bias on expert 0)

and a reduced ``*-small`` variant of each (same E, k, R, payload, bias and capacity rule; smaller T,
H, F with ragged tails) that the oracle finishes in seconds.

Draw order for one workload, from one ``torch.Generator`` seeded with ``seed``:
logits N(0,1) [T,E] fp32 -> bias (per workload) -> x N(0,1) [T,H] -> w_gate N(0,0.02) [E,F,H]
-> w_up N(0,0.02) [E,F,H] -> w_down N(0,0.02) [E,H,F].  x and the weights are drawn in fp32 and
cast to bf16 by torch (round to nearest even).  The bias is added into the logits the router sees.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import torch

__all__ = ["Workload", "WORKLOADS", "get", "make_inputs", "make_weights", "randn_bf16",
           "zipf_log_bias"]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: int            # tokens
    H: int            # hidden size
    E: int            # experts
    k: int            # experts per token
    R: int            # emulated expert-parallel ranks (rank r owns experts [r*E/R, (r+1)*E/R))
    F: int            # SwiGLU intermediate size (d_ff)
    payload: str = "bf16"          # "bf16" or "fp8" (e4m3 + fp32 scale per 128-element block)
    capacity_factor: float = 0.0   # 0 = no drop
    bias: str = "none"             # "none" | "normal0.5" | "zipf1.2" | "hot0+3"
    weight_std: float = 0.02

    @property
    def slots(self) -> int:
        return self.T * self.k

    def describe(self) -> str:
        s = (f"{self.name}: T={self.T} H={self.H} E={self.E} k={self.k} R={self.R} F={self.F} "
             f"payload={self.payload}")
        if self.capacity_factor:
            s += f" cf={self.capacity_factor}"
        if self.bias != "none":
            s += f" bias={self.bias}"
        return s


_FULL = [
    Workload("tiny", 128, 256, 8, 2, 4, 512),
    Workload("decode", 128, 4096, 8, 2, 8, 14336),
    Workload("train", 4096, 4096, 8, 2, 8, 14336, bias="normal0.5"),
    Workload("finegrained", 4096, 7168, 256, 8, 32, 2048, payload="fp8", bias="zipf1.2"),
    Workload("skewed", 16384, 7168, 128, 2, 16, 2048, capacity_factor=1.25, bias="hot0+3"),
]
_SMALL = [
    Workload("decode-small", 128, 512, 8, 2, 8, 704),
    Workload("train-small", 1000, 768, 8, 2, 8, 1024, bias="normal0.5"),
    Workload("finegrained-small", 300, 1024, 256, 8, 32, 256, payload="fp8", bias="zipf1.2"),
    Workload("skewed-small", 2048, 512, 128, 2, 16, 320, capacity_factor=1.25, bias="hot0+3"),
]
# Profiler-sized: the train shapes (H=4096, F=14336) with two experts and k=1, so the expert FFN is
# tensor-bound like train's (about 1000 rows per expert) while all buffers fit in about 1 GB.
_PROFILE = [
    Workload("train-e2", 2048, 4096, 2, 1, 2, 14336),
    # the skewed shapes (H=7168, F=2048, about 256 rows per expert) with 16 experts: the expert
    # FFN streams its weights like skewed's while the buffers stay at about 2 GB
    Workload("skewed-e16", 2048, 7168, 16, 2, 16, 2048),
]
WORKLOADS: Dict[str, Workload] = {w.name: w for w in _FULL + _SMALL + _PROFILE}


def get(name: str) -> Workload:
    return WORKLOADS[name]


def zipf_log_bias(E: int, s: float, gen: torch.Generator) -> torch.Tensor:
    """bias_e = ln p_{pi(e)} - mean, p_i proportional to i^-s (i = 1..E), pi a seeded permutation."""
    ranks = torch.arange(1, E + 1, dtype=torch.float64)
    logp = -s * torch.log(ranks)
    logp = logp - torch.logsumexp(logp, 0)
    perm = torch.randperm(E, generator=gen, device=gen.device).cpu()
    bias = logp[perm]
    return (bias - bias.mean()).to(torch.float32)


def _bias(w: Workload, gen: torch.Generator) -> Optional[torch.Tensor]:
    dev = gen.device
    if w.bias == "none":
        return None
    if w.bias == "normal0.5":
        return torch.randn(w.E, generator=gen, device=dev, dtype=torch.float32) * 0.5
    if w.bias == "zipf1.2":
        return zipf_log_bias(w.E, 1.2, gen).to(dev)
    if w.bias == "hot0+3":
        b = torch.zeros(w.E, dtype=torch.float32, device=dev)
        b[0] = 3.0
        return b
    raise ValueError(f"unknown bias {w.bias}")


def randn_bf16(shape, gen: torch.Generator, std: float = 1.0) -> torch.Tensor:
    """N(0, std^2) drawn in fp32 on the generator's device, cast to bf16 (round to nearest even)."""
    t = torch.randn(shape, generator=gen, device=gen.device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(torch.bfloat16)


def make_inputs(w: Workload, seed: int = 0, device: str = "cpu", weights: bool = True):
    """Router logits (bias included), token activations and, optionally, expert weights.

    Returns a dict of tensors on ``device``: ``logits`` fp32 [T,E], ``x`` bf16 [T,H] and, when
    ``weights`` is true, ``w_gate`` / ``w_up`` bf16 [E,F,H] and ``w_down`` bf16 [E,H,F].
    """
    gen = torch.Generator(device=device).manual_seed(seed)
    logits = torch.randn((w.T, w.E), generator=gen, device=device, dtype=torch.float32)
    b = _bias(w, gen)
    if b is not None:
        logits = logits + b[None, :]
    x = randn_bf16((w.T, w.H), gen)
    out = {"logits": logits.contiguous(), "x": x}
    if weights:
        out.update(make_weights(w, gen))
    return out


def make_weights(w: Workload, gen: torch.Generator):
    return {
        "w_gate": randn_bf16((w.E, w.F, w.H), gen, w.weight_std),
        "w_up": randn_bf16((w.E, w.F, w.H), gen, w.weight_std),
        "w_down": randn_bf16((w.E, w.H, w.F), gen, w.weight_std),
    }


def random_topk(T: int, E: int, k: int, gen: torch.Generator) -> torch.Tensor:
    """k distinct expert ids per token, uniformly at random (int32 [T,k])."""
    keys = torch.rand((T, E), generator=gen, device=gen.device)
    return keys.argsort(dim=1)[:, :k].to(torch.int32).contiguous()


def random_weights_rows(T: int, k: int, gen: torch.Generator) -> torch.Tensor:
    """Positive per-slot weights (fp32 [T,k]) for stage-level combine inputs."""
    return torch.rand((T, k), generator=gen, device=gen.device, dtype=torch.float32).contiguous()


def l2_flush_bytes() -> int:
    """Size of the scratch write that evicts the B200's 126 MB L2 between timed iterations."""
    return 256 * 1024 * 1024



def make_ep_inputs(w: Workload, ranks: int, seed: int = 0, device: str = "cpu"):
    """Inputs of an expert-parallel step over ``ranks`` ranks: every rank has its own T tokens
    (``make_inputs`` with seed ``1000 * seed + 1 + rank``, weights left out) and the expert weights
    are those of ``make_inputs(w, seed)``.  Returns ``{"logits": [per rank], "x": [per rank],
    "w_gate", "w_up", "w_down"}``; rank r keeps experts [r*E/ranks, (r+1)*E/ranks) of the weights."""
    full = make_inputs(w, seed=seed, device=device, weights=True)
    per = [make_inputs(w, seed=1000 * seed + 1 + r, device=device, weights=False)
           for r in range(ranks)]
    return {"logits": [p["logits"] for p in per], "x": [p["x"] for p in per],
            "w_gate": full["w_gate"], "w_up": full["w_up"], "w_down": full["w_down"]}
