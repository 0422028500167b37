"""Seeded synthetic inputs and the named workloads.

This module holds no attention arithmetic: it only draws the random tensors
that both the CUDA library and the fp64 oracle consume, so that the two sides
see identical values.  Recipe: a ``torch.Generator`` seeded with ``seed`` on
the device the tensors are made on draws Q, K, V, dO in that order with
``torch.randn(B, H, N, d, dtype=float32)``; Q is multiplied by ``q_mult``
before the cast to the storage dtype.  The oracle receives the cast values,
upcast exactly to float64.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    Nq: int
    Nk: int
    d: int
    causal: bool
    dtype: str = "bf16"
    q_mult: float = 1.0
    seed: int = 0
    decode: bool = False
    extra: dict = field(default_factory=dict, compare=False)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def fwd_flops(self) -> float:
        f = 4.0 * self.B * self.H * self.Nq * self.Nk * self.d
        return f / 2 if self.causal else f

    @property
    def bwd_flops(self) -> float:
        return 2.5 * self.fwd_flops

    def describe(self) -> str:
        c = "causal" if self.causal else "non-causal"
        return (f"B{self.B} H{self.H} Nq{self.Nq} Nk{self.Nk} d{self.d} "
                f"{self.dtype} {c}" + (f" Q×{self.q_mult:g}" if self.q_mult != 1 else ""))


# The five named workloads.
TINY_FP32 = Workload("tiny_fp32", 1, 1, 128, 128, 64, False, "fp32")
TINY_BF16 = Workload("tiny_bf16", 1, 1, 128, 128, 64, False, "bf16")
MEDIUM = Workload("b4h16n1024d64", 4, 16, 1024, 1024, 64, False, "bf16")
CAUSAL_2K = Workload("b8h16n2048d128_causal", 8, 16, 2048, 2048, 128, True, "bf16")
LONG_16K = Workload("b1h32n16384d128_causal_q3", 1, 32, 16384, 16384, 128, True, "bf16", q_mult=3.0)
# the causal 2K workload in fp16 (timed like bf16; a parity case as well)
CAUSAL_2K_FP16 = Workload("b8h16n2048d128_causal_fp16", 8, 16, 2048, 2048, 128, True, "fp16")
DECODE_32K = Workload("decode_b32h32nk32768d128", 32, 32, 1, 32768, 128, False, "bf16", decode=True)

ALL = [TINY_FP32, TINY_BF16, MEDIUM, CAUSAL_2K, LONG_16K, DECODE_32K]

TORCH_DTYPES = {"fp32": torch.float32, "bf16": torch.bfloat16, "fp16": torch.float16}


def make_inputs(w: Workload, device="cpu", with_grad: bool = True):
    """Draw (Q, K, V, dO) for a workload; dO is None for decode or when
    ``with_grad`` is False.  Shapes [B, H, N, d], contiguous."""
    return make_tensors(w.B, w.H, w.Nq, w.Nk, w.d, w.dtype, seed=w.seed,
                        q_mult=w.q_mult, device=device,
                        with_grad=with_grad and not w.decode)


def make_tensors(B, H, Nq, Nk, d, dtype="bf16", seed=0, q_mult=1.0,
                 device="cpu", with_grad=True):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    dt = TORCH_DTYPES[dtype]

    def draw(n):
        return torch.randn(B, H, n, d, dtype=torch.float32, device=device, generator=g)

    q = draw(Nq)
    if q_mult != 1.0:
        q = q * q_mult
    k = draw(Nk)
    v = draw(Nk)
    do = draw(Nq) if with_grad else None
    cast = lambda t: None if t is None else t.to(dt).contiguous()
    return cast(q), cast(k), cast(v), cast(do)
