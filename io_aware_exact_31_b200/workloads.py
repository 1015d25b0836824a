"""Seeded synthetic workloads for attention (inputs only; no attention arithmetic).

The same generator feeds the CUDA path, the fp64 oracle and the benchmark, so
both sides see bit-identical bf16 inputs.  Recipe: one CPU ``torch.Generator``
seeded with ``seed`` draws Q, K, V and then (for backward workloads) dO, in
that order, each as i.i.d. N(0, 1) float32 of shape [B, H, N, d], rounded to
bf16 (round-to-nearest-even).  A workload with ``input_scale`` 2 multiplies
the bf16 tensors by 2, which is exact.

Shapes follow the pages' workloads: the 8-head, 64-dim, 1024-token causal
transformer of downcodes.com "triton transformer" (usage section), the
4k-token example of aiunderstanding.org "FlashAttention" (deep dive), and the
16k context of systems-analysis.info "FlashAttention-2 (VI)" (performance
section).  No dataset is involved.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    causal: bool
    input_scale: float = 1.0
    backward: bool = False

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def fwd_flops(self) -> float:
        """4*B*H*N^2*d, halved when causal (the counting convention, not exact)."""
        f = 4.0 * self.B * self.H * self.N * self.N * self.d
        return f / 2 if self.causal else f

    @property
    def bwd_flops(self) -> float:
        return 2.5 * self.fwd_flops

    @property
    def fwd_bytes(self) -> int:
        """Algorithmic HBM bytes of the forward: read Q, K, V, write O (bf16) and LSE (fp32)."""
        n = self.B * self.H * self.N
        return 4 * n * self.d * 2 + n * 4

    @property
    def bwd_bytes(self) -> int:
        """Read Q, K, V, O, dO, LSE; write dQ, dK, dV (bf16).  D is internal."""
        n = self.B * self.H * self.N
        return 8 * n * self.d * 2 + n * 4

    def describe(self) -> str:
        c = "causal" if self.causal else "non-causal"
        s = f"B={self.B} H={self.H} N={self.N} d={self.d} {c} scale=1/sqrt({self.d})"
        if self.input_scale != 1.0:
            s += f" inputs x{self.input_scale:g}"
        return s


# The five workloads: tiny, the 8-head/64-dim/1024-token causal transformer,
# 4k tokens at d=128, a 16k causal context with a widened score range, and a
# causal forward+backward case.
WORKLOADS = {
    "tiny_n256_d64": Workload("tiny_n256_d64", 1, 1, 256, 64, False),
    "transformer_h8_n1024_d64_causal": Workload("transformer_h8_n1024_d64_causal", 1, 8, 1024,
                                                64, True),
    "b4_h16_n4096_d128": Workload("b4_h16_n4096_d128", 4, 16, 4096, 128, False),
    "h16_n16384_d128_causal_x2": Workload("h16_n16384_d128_causal_x2", 1, 16, 16384, 128,
                                          True, input_scale=2.0),
    "b4_h16_n2048_d64_causal_bwd": Workload("b4_h16_n2048_d64_causal_bwd", 4, 16, 2048, 64,
                                            True, backward=True),
}


def make_inputs(B: int, H: int, N: int, d: int, seed: int = 0, input_scale: float = 1.0,
                with_dO: bool = False):
    """Q, K, V (and dO) as contiguous bf16 CPU tensors [B, H, N, d]."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    names = ["Q", "K", "V"] + (["dO"] if with_dO else [])
    out = {}
    for n in names:
        t = torch.randn(B, H, N, d, generator=g, dtype=torch.float32).to(torch.bfloat16)
        if input_scale != 1.0:
            t = t * input_scale
        out[n] = t.contiguous()
    return out


def workload_inputs(w: Workload, seed: int = 0):
    return make_inputs(w.B, w.H, w.N, w.d, seed=seed, input_scale=w.input_scale,
                       with_dO=w.backward)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """The raw bf16 bit patterns of a CPU tensor as a uint16 numpy array."""
    assert t.dtype == torch.bfloat16
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)
