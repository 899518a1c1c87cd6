"""Seeded synthetic workloads for the MoE route / layout / dispatch / combine path.

This module only draws inputs.  It holds none of the method's arithmetic, so
both the CUDA path and the CPU oracle can be fed from it.

The five workloads follow the shapes and value distributions of the pages'
regimes ("GPU MoE all-to-all", section "Latency-bound at decode,
bandwidth-bound at prefill" and section "Routing skew turns a symmetric
collective asymmetric"; "19. All-to-all", section "Why Qwen3.8's 512 experts is
a systems statement" for the 512-expert, 10 routed + 1 shared layout):

  tiny        T=256   H=128  E=8   R=4  k=2   identity experts
  prefill     T=4096  H=4096 E=128 R=16 k=8   expert e scales rows by (e+1)/E
  decode      T=128   H=7168 E=256 R=32 k=8   per-expert bias U(-0.1, 0.1)
  skewed      T=32768 H=7168 E=256 R=32 k=8   Zipf(1.2) popularity offsets,
                                              capacity factor 1.2 or dropless
  finegrained T=65536 H=2048 E=512 R=64 k=10  + shared expert, FP8 dispatch,
                                              residual add

Recipe (seed 0 unless stated; one torch CPU generator, draws in this order):
  1. x      = randn(T, H) in fp32, rounded to bf16 (nearest even);
  2. logits = randn(T, E) in fp32; skewed adds 2*ln(p_e) with
              p_e = (e+1)^-1.2 / sum_e' (e'+1)^-1.2 (computed in fp64, rounded
              to fp32, then one fp32 add);
  3. bias   = rand(E) * 0.2 - 0.1 in fp32 (decode only);
  4. shared = randn(T, H) in fp32, rounded to bf16 (workloads with a shared
              expert): the always-on expert's output, a tensor of its own so
              the combine's shared and residual operands differ.
Each draw comes after the ones before it, so adding a later one leaves the
earlier inputs unchanged.
"""
from __future__ import annotations

import dataclasses
import math
from fractions import Fraction
from typing import Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: int
    H: int
    E: int
    R: int
    k: int
    capacity_factor: Optional[Fraction] = None  # None: dropless
    align: int = 1
    bias: bool = False
    zipf_s: Optional[float] = None
    fp8: bool = False
    shared: bool = False
    residual: bool = False
    expert: str = "identity"  # identity | scale | dequant (test stand-ins)
    renorm: bool = True
    seed: int = 0

    @property
    def capacity(self) -> int:
        """Per-expert slots C = ceil(cf * T * k / E); 0 means dropless."""
        if self.capacity_factor is None:
            return 0
        return max(1, math.ceil(Fraction(self.capacity_factor) * self.T * self.k / self.E))

    @property
    def rows(self) -> int:
        """Rows of the dispatched buffer (static bound, no count read-back)."""
        if self.capacity:
            return self.E * self.capacity
        return self.T * self.k + self.E * (self.align - 1)

    @property
    def capacity_src(self) -> int:
        """Per-(source shard, expert) slots for the per-source-rank layout:
        C = ceil(cf * Ts * k / E) with Ts = ceil(T/R) tokens per shard; 0 means
        dropless."""
        if self.capacity_factor is None:
            return 0
        ts = -(-self.T // self.R) if self.T > 0 else 1
        return max(1, math.ceil(Fraction(self.capacity_factor) * ts * self.k / self.E))

    @property
    def rows_src(self) -> int:
        """Rows of the per-source-rank layout (segments per (rank, shard, expert))."""
        if self.capacity_src:
            return self.R * self.E * self.capacity_src
        return self.T * self.k + self.R * self.E * (self.align - 1)

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    def describe(self) -> str:
        mode = f"capacity C={self.capacity}" if self.capacity else "dropless"
        extra = []
        if self.bias:
            extra.append("bias U(-0.1,0.1)")
        if self.zipf_s:
            extra.append(f"Zipf({self.zipf_s}) offsets")
        if self.fp8:
            extra.append("FP8 e4m3 dispatch, per-128 scales")
        if self.shared:
            extra.append("shared expert")
        if self.residual:
            extra.append("residual")
        return (f"{self.name}: T={self.T} H={self.H} E={self.E} R={self.R} k={self.k} {mode}"
                + ("" if not extra else ", " + ", ".join(extra)))


WORKLOADS = {
    "tiny": Workload("tiny", T=256, H=128, E=8, R=4, k=2),
    "prefill": Workload("prefill", T=4096, H=4096, E=128, R=16, k=8, expert="scale"),
    "decode": Workload("decode", T=128, H=7168, E=256, R=32, k=8, bias=True),
    "skewed_capacity": Workload("skewed_capacity", T=32768, H=7168, E=256, R=32, k=8,
                                zipf_s=1.2, capacity_factor=Fraction(6, 5)),
    "skewed_dropless": Workload("skewed_dropless", T=32768, H=7168, E=256, R=32, k=8,
                                zipf_s=1.2),
    "finegrained": Workload("finegrained", T=65536, H=2048, E=512, R=64, k=10, fp8=True,
                            shared=True, residual=True, expert="dequant"),
}


@dataclasses.dataclass
class Inputs:
    x: torch.Tensor            # bf16 [T, H]
    logits: torch.Tensor       # fp32 [T, E]
    bias: Optional[torch.Tensor]  # fp32 [E] or None
    shared: Optional[torch.Tensor] = None  # bf16 [T, H] shared-expert output, or None


def zipf_offsets(E: int, s: float) -> torch.Tensor:
    """2 * ln(p_e), p_e proportional to (e+1)^-s; fp64 then rounded to fp32."""
    e = torch.arange(1, E + 1, dtype=torch.float64)
    w = e.pow(-s)
    p = w / w.sum()
    return (2.0 * torch.log(p)).to(torch.float32)


def make_inputs(w: Workload, seed: Optional[int] = None) -> Inputs:
    """Draw x, logits, bias and the shared-expert output on the CPU, in that
    order, from one generator."""
    g = torch.Generator().manual_seed(w.seed if seed is None else seed)
    x = torch.randn(w.T, w.H, generator=g, dtype=torch.float32).to(torch.bfloat16)
    logits = torch.randn(w.T, w.E, generator=g, dtype=torch.float32)
    if w.zipf_s:
        logits = logits + zipf_offsets(w.E, w.zipf_s)
    bias = None
    if w.bias:
        bias = torch.rand(w.E, generator=g, dtype=torch.float32) * 0.2 - 0.1
    shared = None
    if w.shared:
        shared = torch.randn(w.T, w.H, generator=g, dtype=torch.float32).to(torch.bfloat16)
        shared = shared.contiguous()
    return Inputs(x=x.contiguous(), logits=logits.contiguous(), bias=bias, shared=shared)


def bf16_bits(t: torch.Tensor):
    """bf16 tensor -> numpy uint16 bit patterns (CPU copy)."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view("uint16")


def bits_to_bf16(a) -> torch.Tensor:
    import numpy as np
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
