"""Seeded synthetic inputs for the MoE layer with zero-computation experts.

This module only draws random numbers and lays them out.  It holds none of the
layer's arithmetic (no router, softmax, top-K or FFN), so the CUDA path and
the fp64 oracle can both take their inputs from it.

Shapes and distributions follow the five workloads the layer is measured on:
x ~ N(0, 1), expert and router weights ~ N(0, w_std), all rounded once to
bf16; the expert bias b ~ U[-0.1, 0.1] in fp32, plus one shift `delta` added
to every zero-computation expert's entry so that a stated share of all picks
lands on zero experts.  The skewed workload also gives each FFN expert a
Zipf(s) router-logit offset (offset_i = -s * ln(rank_i)).

Because |b| (up to 0.1) is far above a typical softmax score (~1/E), that
bias decides most picks and the FFN load is concentrated on a few dozen
experts.  Two balanced companions of the LongCat-shaped workloads
(``prefill_balanced``, ``decode_balanced``: same seeds, x and W_r) set the
FFN experts' bias to zero instead, so the softmax scores decide among the
FFN experts and every expert gets about the same expected load -- the state
the bias controller steers towards.

Where the numbers come from:
  * x, W_r, b and the Zipf ranks come from a CPU ``torch.Generator`` seeded
    with the workload seed, in that order.  Routing depends only on these, so
    it is identical on every machine, and the bias shifts below (found on a
    CPU) hold on the GPU too.
  * The FFN weights are drawn expert by expert (W_gate[e], W_up[e],
    W_down[e]) by a generator on the device the tensors are made on, seeded
    with ``seed + 1``.  They differ between CPU and CUDA; a parity test always
    draws them once and hands the same tensors to both sides.
"""
from __future__ import annotations

import json
import os
from dataclasses import dataclass, field, replace
from typing import Optional

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    T: int          # tokens
    d: int          # model width
    N: int          # SwiGLU FFN experts
    Z: int          # zero-computation (identity) experts
    K: int          # experts picked per token
    I: int          # FFN intermediate width
    w_std: float    # std of W_r, W_gate, W_up, W_down
    seed: int
    zero_frac: Optional[float] = None   # target share of picks on zero experts
    zipf_s: Optional[float] = None      # Zipf exponent of the logit offset
    delta: float = 0.0                  # shift added to the zero experts' bias
    bias: str = "random"                # b0: "random" U[-0.1, 0.1], or "zero"

    @property
    def E(self) -> int:
        return self.N + self.Z


# Bias shifts found by bisection with the fp64 router so that the share of
# zero-expert picks over all T*K picks meets `zero_frac` (within 0.005).
# Written by oracle/calibrate_bias_shift.py, re-checked by
# tests/test_workloads.py.
_DELTA_FILE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "bias_shift.json")
_DELTA = {}
if os.path.exists(_DELTA_FILE):
    with open(_DELTA_FILE) as _f:
        _DELTA = json.load(_f)

WORKLOADS = {
    w.name: w
    for w in [
        Workload("tiny", T=256, d=256, N=8, Z=4, K=2, I=512, w_std=0.02, seed=0),
        Workload("small", T=4096, d=2048, N=64, Z=32, K=6, I=1024, w_std=0.02, seed=1),
        Workload("prefill", T=16384, d=6144, N=512, Z=256, K=12, I=2048, w_std=0.01,
                 seed=2, zero_frac=0.30),
        Workload("decode", T=64, d=6144, N=512, Z=256, K=12, I=2048, w_std=0.01,
                 seed=3, zero_frac=0.40),
        Workload("prefill_balanced", T=16384, d=6144, N=512, Z=256, K=12, I=2048,
                 w_std=0.01, seed=2, zero_frac=0.30, bias="zero"),
        Workload("decode_balanced", T=64, d=6144, N=512, Z=256, K=12, I=2048, w_std=0.01,
                 seed=3, zero_frac=0.40, bias="zero"),
        Workload("skewed20", T=32768, d=4096, N=256, Z=128, K=8, I=1536, w_std=0.02,
                 seed=4, zero_frac=0.20, zipf_s=1.1),
        Workload("skewed40", T=32768, d=4096, N=256, Z=128, K=8, I=1536, w_std=0.02,
                 seed=4, zero_frac=0.40, zipf_s=1.1),
        Workload("skewed60", T=32768, d=4096, N=256, Z=128, K=8, I=1536, w_std=0.02,
                 seed=4, zero_frac=0.60, zipf_s=1.1),
    ]
}
WORKLOADS = {k: replace(w, delta=_DELTA.get(k, 0.0)) for k, w in WORKLOADS.items()}


def get(workload: str, **overrides) -> Workload:
    """The named workload, optionally with fields replaced (e.g. T=512)."""
    return replace(WORKLOADS[workload], **overrides)


@dataclass
class RoutingInputs:
    x: torch.Tensor                      # [T, d] bf16
    W_r: torch.Tensor                    # [E, d] bf16
    b0: torch.Tensor                     # [E] fp32, before the zero-expert shift
    logit_offset: Optional[torch.Tensor] = None   # [E] fp32 or None

    def bias(self, N: int, delta: float) -> torch.Tensor:
        """b = b0 + delta on the zero experts (rows N..E-1)."""
        b = self.b0.clone()
        b[N:] += delta
        return b


def routing_inputs(w: Workload, T: Optional[int] = None) -> RoutingInputs:
    """x, W_r, b0 (and the Zipf offset) on the CPU, from the workload seed.

    ``T`` below the workload's T gives the first T rows of the same x.
    """
    g = torch.Generator().manual_seed(w.seed)
    x = torch.randn(w.T, w.d, generator=g, dtype=torch.float32).to(torch.bfloat16)
    W_r = (torch.randn(w.E, w.d, generator=g, dtype=torch.float32) * w.w_std).to(torch.bfloat16)
    b0 = torch.rand(w.E, generator=g, dtype=torch.float32) * 0.2 - 0.1
    if w.bias == "zero":        # drawn all the same, so later draws do not move
        b0 = torch.zeros_like(b0)
    off = None
    if w.zipf_s is not None:
        rank = torch.randperm(w.N, generator=g) + 1           # rank 1..N per FFN expert
        off = torch.zeros(w.E, dtype=torch.float32)
        off[: w.N] = -w.zipf_s * torch.log(rank.to(torch.float64)).to(torch.float32)
    if T is not None and T < w.T:
        x = x[:T].contiguous()
    return RoutingInputs(x=x, W_r=W_r, b0=b0, logit_offset=off)


@dataclass
class ExpertWeights:
    W_gate: torch.Tensor   # [N, I, d] bf16
    W_up: torch.Tensor     # [N, I, d] bf16
    W_down: torch.Tensor   # [N, d, I] bf16


def expert_weights(w: Workload, device="cpu") -> ExpertWeights:
    """SwiGLU expert weights, drawn expert by expert on ``device``."""
    dev = torch.device(device)
    g = torch.Generator(device=dev).manual_seed(w.seed + 1)
    Wg = torch.empty(w.N, w.I, w.d, dtype=torch.bfloat16, device=dev)
    Wu = torch.empty(w.N, w.I, w.d, dtype=torch.bfloat16, device=dev)
    Wd = torch.empty(w.N, w.d, w.I, dtype=torch.bfloat16, device=dev)
    for e in range(w.N):
        Wg[e].normal_(0.0, w.w_std, generator=g)
        Wu[e].normal_(0.0, w.w_std, generator=g)
        Wd[e].normal_(0.0, w.w_std, generator=g)
    return ExpertWeights(W_gate=Wg, W_up=Wu, W_down=Wd)


def tokens_sample(T: int, n: int, seed: int) -> torch.Tensor:
    """A seeded, sorted sample of n distinct token rows out of T."""
    g = torch.Generator().manual_seed(10_000 + seed)
    n = min(n, T)
    return torch.randperm(T, generator=g)[:n].sort().values
