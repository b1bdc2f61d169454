"""Seeded synthetic inputs for attention, shared by the oracle tests, the GPU
parity tests and the benchmark.

This module only draws random numbers and rounds them to the working dtype.
It holds none of the attention arithmetic, so neither side of a parity test
can borrow a step of the method from here.

Recipe (one call per workload): a CPU ``torch.Generator`` seeded with the
workload's seed draws Q, K, V and dO, in that order, as fp32 standard normals
scaled by each tensor's standard deviation. For a bf16 workload every tensor
is then rounded to bf16, and both the GPU path and the float64 oracle see
exactly those rounded values, so input quantisation is never counted as error.
"""
from __future__ import annotations

import dataclasses
import math

import torch

__all__ = ["Workload", "WORKLOADS", "workload", "make_inputs", "make_small"]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    n: int           # query positions
    m: int           # key positions
    d: int           # query/key width
    dv: int          # value width
    dtype: str       # "f32" or "bf16"
    causal: bool
    seed: int
    std_qk: float = 1.0
    std_vo: float = 1.0
    doc: str = ""

    @property
    def scale(self) -> float:
        # Scores are divided by the square root of the query/key width.
        return 1.0 / math.sqrt(self.d)

    def bwd_flops(self) -> float:
        """Counted backward FLOPs: 2.5x the forward's two matmuls, halved when causal."""
        f = 2.5 * 4.0 * self.B * self.H * self.n * self.m * self.d
        return f / 2.0 if self.causal else f

    def fwd_flops(self) -> float:
        f = 4.0 * self.B * self.H * self.n * self.m * self.d
        return f / 2.0 if self.causal else f


WORKLOADS = {
    "single_head_f32_64": Workload(
        "single_head_f32_64", 1, 1, 64, 64, 64, 64, "f32", False, 1,
        doc="single head, no batch: 64x64 fp32, non-causal"),
    "causal_b4h16_n1024_d64": Workload(
        "causal_b4h16_n1024_d64", 4, 16, 1024, 1024, 64, 64, "bf16", True, 2,
        doc="B=4 H=16 N=1024 d=64 bf16 causal"),
    "causal_b2h32_n4096_d128": Workload(
        "causal_b2h32_n4096_d128", 2, 32, 4096, 4096, 128, 128, "bf16", True, 3,
        doc="B=2 H=32 N=4096 d=128 bf16 causal (headline)"),
    "cross_b8h16_n512_m2048_d64": Workload(
        "cross_b8h16_n512_m2048_d64", 8, 16, 512, 2048, 64, 64, "bf16", False, 4,
        std_qk=3.0, std_vo=1.0,
        doc="cross-attention B=8 H=16 n=512 m=2048 d=64 bf16, Q,K ~ N(0,9)"),
    "causal_b4h16_n1024_d64_f32": Workload(
        "causal_b4h16_n1024_d64_f32", 4, 16, 1024, 1024, 64, 64, "f32", True, 6,
        doc="B=4 H=16 N=1024 d=64 fp32 causal (the fp32 tensor-core path)"),
    "causal_b1h32_n16384_d128": Workload(
        "causal_b1h32_n16384_d128", 1, 32, 16384, 16384, 128, 128, "bf16", True, 5,
        doc="long context B=1 H=32 N=16384 d=128 bf16 causal"),
}


def workload(name: str) -> Workload:
    return WORKLOADS[name]


def _round(t: torch.Tensor, dtype: str) -> torch.Tensor:
    if dtype == "bf16":
        return t.to(torch.bfloat16)
    if dtype == "f32":
        return t
    raise ValueError(dtype)


def make_inputs(w: Workload, seed: int | None = None):
    """Return (Q, K, V, dO) as CPU tensors of the workload's dtype, [B,H,N,d]."""
    g = torch.Generator().manual_seed(w.seed if seed is None else seed)
    q = torch.randn((w.B, w.H, w.n, w.d), generator=g, dtype=torch.float32) * w.std_qk
    k = torch.randn((w.B, w.H, w.m, w.d), generator=g, dtype=torch.float32) * w.std_qk
    v = torch.randn((w.B, w.H, w.m, w.dv), generator=g, dtype=torch.float32) * w.std_vo
    do = torch.randn((w.B, w.H, w.n, w.dv), generator=g, dtype=torch.float32) * w.std_vo
    return tuple(_round(t, w.dtype) for t in (q, k, v, do))


def make_small(B, H, n, m, d, dv, dtype="bf16", causal=False, seed=0,
               std_qk=1.0, std_vo=1.0) -> Workload:
    """An ad-hoc workload for tests (ragged and edge shapes)."""
    return Workload(f"adhoc_{B}x{H}x{n}x{m}x{d}x{dv}_{dtype}_{int(causal)}_{seed}",
                    B, H, n, m, d, dv, dtype, causal, seed, std_qk, std_vo)
