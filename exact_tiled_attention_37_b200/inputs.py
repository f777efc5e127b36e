"""Seeded synthetic inputs for the attention workloads.

This module only draws random numbers and casts them; it holds none of the
attention arithmetic, so both the CUDA path's tests/benchmark and the oracle
can be fed from it without sharing any of the method's code.

Recipe: a CPU ``torch.Generator`` seeded with ``1000 + workload index``; the
tensors are drawn in the order Q, K, V, dO, each i.i.d. N(0, 1) in float32 and
then rounded (round-to-nearest-even) to the storage dtype.  The long-context
grouped-query workload multiplies K by 3 in float32 before the cast, which
sharpens the softmax so that the running maximum moves and the rescale path
is exercised.
"""

from __future__ import annotations

import dataclasses
import math

import torch

__all__ = ["Workload", "WORKLOADS", "workload", "make_inputs", "make_random"]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    index: int
    B: int
    Hq: int
    Hkv: int
    N: int
    D: int
    dtype: str            # "bf16" or "fp32"
    causal: tuple         # mask modes run on this workload
    backward: bool
    k_mult: float = 1.0

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    def fwd_flops(self, causal: bool) -> float:
        f = 4.0 * self.B * self.Hq * self.N * self.N * self.D
        return f / 2 if causal else f

    def bwd_flops(self, causal: bool) -> float:
        return 2.5 * self.fwd_flops(causal)


WORKLOADS = (
    Workload("single-head fp32 N=256 D=64", 0, 1, 1, 1, 256, 64, "fp32", (False,), False),
    Workload("MHA B=4 H=16 N=2048 D=128", 1, 4, 16, 16, 2048, 128, "bf16", (False, True), False),
    Workload("MHA fwd+bwd B=2 H=16 N=4096 D=128 causal", 2, 2, 16, 16, 4096, 128, "bf16", (True,), True),
    Workload("GQA B=1 Hq=32 Hkv=8 N=32768 D=128 causal, K x3", 3, 1, 32, 8, 32768, 128, "bf16",
             (True,), False, 3.0),
    Workload("MHA fwd+bwd B=8 H=8 N=8192 D=256", 4, 8, 8, 8, 8192, 256, "bf16", (False,), True),
)


def workload(index: int) -> Workload:
    return WORKLOADS[index]


def _cast(x: torch.Tensor, dtype: str) -> torch.Tensor:
    return x.to(torch.bfloat16) if dtype == "bf16" else x.contiguous()


def make_random(B, Hq, Hkv, N, D, dtype="bf16", seed=0, k_mult=1.0, with_do=True):
    """Q, K, V (and dO) as CPU tensors [B, H, N, D], drawn in that order."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    q = torch.randn((B, Hq, N, D), generator=g, dtype=torch.float32)
    k = torch.randn((B, Hkv, N, D), generator=g, dtype=torch.float32)
    if k_mult != 1.0:
        k = k * k_mult
    v = torch.randn((B, Hkv, N, D), generator=g, dtype=torch.float32)
    out = [_cast(q, dtype), _cast(k, dtype), _cast(v, dtype)]
    if with_do:
        do = torch.randn((B, Hq, N, D), generator=g, dtype=torch.float32)
        out.append(_cast(do, dtype))
    return tuple(out)


def make_inputs(w: Workload, with_do=None):
    """Inputs of a named workload with its own seed (1000 + index)."""
    if with_do is None:
        with_do = w.backward
    return make_random(w.B, w.Hq, w.Hkv, w.N, w.D, w.dtype, 1000 + w.index, w.k_mult, with_do)
