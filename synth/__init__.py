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

Padded workloads also carry the number of valid keys of each batch element
(the key padding mask): either listed, or drawn uniformly from
[pad_min, m] by a generator seeded with seed + 7919.
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
    pad_min: int = 0                 # > 0: key lengths drawn from [pad_min, m]
    lengths: tuple | None = None     # explicit key lengths, one per batch element

    def key_len(self):
        """Valid keys per batch element (list of B ints), or None unpadded."""
        if self.lengths is not None:
            return [int(x) for x in self.lengths]
        if self.pad_min <= 0:
            return None
        g = torch.Generator().manual_seed(self.seed + 7919)
        return [int(x) for x in torch.randint(self.pad_min, self.m + 1, (self.B,), generator=g)]

    def _pairs(self) -> float:
        """Unmasked (query, key) pairs summed over the batch, per head. The
        unpadded count keeps the n*m/2 convention for causal workloads."""
        kl = self.key_len()
        if kl is None:
            p = self.B * self.n * self.m
            return p / 2.0 if self.causal else float(p)
        total = 0
        for L in kl:
            if self.causal:
                total += sum(min(i + 1, L) for i in range(self.n))
            else:
                total += self.n * L
        return float(total)

    @property
    def scale(self) -> float:
        # Scores are divided by the square root of the query/key width.
        return 1.0 / math.sqrt(self.d)

    def bwd_flops(self) -> float:
        """Counted backward FLOPs: 2.5x the forward's two matmuls, halved when
        causal; with a padding mask, over the unmasked pairs only."""
        return 2.5 * 4.0 * self.H * self.d * self._pairs()

    def fwd_flops(self) -> float:
        return 4.0 * self.H * self.d * self._pairs()

    def head_bwd_flops(self, b: int) -> float:
        """Counted backward FLOPs of one (batch element b, head) problem."""
        kl = self.key_len()
        if kl is None:
            return self.bwd_flops() / (self.B * self.H)
        L = kl[b]
        pairs = sum(min(i + 1, L) for i in range(self.n)) if self.causal else self.n * L
        return 2.5 * 4.0 * self.d * pairs


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
    "padded_b8h16_n1024_d64": Workload(
        "padded_b8h16_n1024_d64", 8, 16, 1024, 1024, 64, 64, "bf16", False, 7, pad_min=128,
        doc="B=8 H=16 N=1024 d=64 bf16 with a key padding mask: valid keys per batch "
            "element uniform in [128, 1024]"),
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
               std_qk=1.0, std_vo=1.0, lengths=None) -> Workload:
    """An ad-hoc workload for tests (ragged and edge shapes); ``lengths``:
    optional key lengths, one per batch element."""
    tag = "" if lengths is None else "_pad" + "-".join(str(int(x)) for x in lengths)
    return Workload(f"adhoc_{B}x{H}x{n}x{m}x{d}x{dv}_{dtype}_{int(causal)}_{seed}{tag}",
                    B, H, n, m, d, dv, dtype, causal, seed, std_qk, std_vo,
                    lengths=None if lengths is None else tuple(int(x) for x in lengths))
