"""Seeded synthetic inputs and the workload table.

This module holds none of the attention arithmetic: it only draws random
tensors and lists shapes.  It is the one module that both the CUDA path's tests
and the fp64 oracle consume, so that both see bit-identical inputs.

Shapes follow the NAT / DiNAT pages: stage resolutions 56/28/14/7 for a 224x224
image with patch size 4, heads (2, 4, 8, 16) with embed_dim 64 doubling per
stage so the head dim is 32 in every stage ("Dilated Neighborhood Attention
Transformer", DinatConfig defaults), kernel size 7, and per-stage dilations
[[1, 8, 1], [1, 4, 1, 4], [1, 2, 1, 2, 1, 2], [1, 1, 1, 1, 1]] (same page, and
the gitcode DiNAT article's stage table).  The segmentation-scale and k=13
shapes stand in for the downstream (ADE20K / COCO) use the pages report; no
dataset is read.

Value recipe: q, k, v ~ N(0, 1) and rpb ~ N(0, 0.02), drawn in fp32 from a CPU
``torch.Generator`` in the order q, k, v, rpb, then rounded to the workload
dtype (round-to-nearest-even, ``Tensor.to``).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

DTYPES = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


@dataclass(frozen=True)
class Shape:
    B: int
    heads: int
    H: int
    W: int
    D: int
    k: int
    d: int
    dtype: str  # "f32" | "f16" | "bf16"
    seed: int

    @property
    def queries_heads(self) -> int:
        return self.B * self.heads * self.H * self.W

    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    def algorithmic_bytes(self) -> int:
        """q, k, v read once + out written once + the bias table."""
        e = self.elem_bytes()
        return 4 * self.B * self.heads * self.H * self.W * self.D * e + self.heads * (2 * self.k - 1) ** 2 * e

    def useful_flops(self) -> int:
        """2*k^2*D for q.k plus 2*k^2*D for p.v, per query and head."""
        return 4 * self.B * self.heads * self.H * self.W * self.k * self.k * self.D

    def describe(self) -> str:
        return (f"B={self.B} heads={self.heads} H={self.H} W={self.W} D={self.D} "
                f"k={self.k} d={self.d} {self.dtype}")


@dataclass(frozen=True)
class Workload:
    name: str
    shapes: tuple[Shape, ...] = field(default_factory=tuple)
    note: str = ""


def _sweep() -> tuple[Shape, ...]:
    out = []
    for j, (heads, L, d) in enumerate([(4, 28, 1), (4, 28, 4), (8, 14, 1), (8, 14, 2), (16, 7, 1)]):
        out.append(Shape(128, heads, L, L, 32, 7, d, "bf16", 300 + j))
    return tuple(out)


def _seg() -> tuple[Shape, ...]:
    out = []
    for j, (k, d) in enumerate([(13, 1), (13, 8), (7, 1)]):
        out.append(Shape(2, 4, 128, 128, 32, k, d, "bf16", 400 + j))
    return tuple(out)


WORKLOADS: dict[str, Workload] = {
    "tiny_fp32": Workload("tiny_fp32", (Shape(1, 2, 14, 14, 32, 7, 1, "f32", 0),),
                          "tiny NA2D fp32, parity only"),
    "nat_tiny_s1_fp16": Workload("nat_tiny_s1_fp16", (Shape(32, 2, 56, 56, 32, 7, 1, "f16", 1),),
                                 "NAT-Tiny stage-1 NA2D, fp16, fp32 accumulate"),
    "dinat_s1_bf16": Workload("dinat_s1_bf16", (Shape(32, 2, 56, 56, 32, 7, 8, "bf16", 2),),
                              "DiNAT stage-1 dilated NA2D (window span 56), bf16"),
    "dinat_sweep_bf16": Workload("dinat_sweep_bf16", _sweep(), "DiNAT stage sweep, bf16, B=128"),
    "seg_bf16": Workload("seg_bf16", _seg(), "segmentation-scale NA2D, bf16, B=2"),
}

# the workload the headline throughput is quoted on
HEADLINE = "nat_tiny_s1_fp16"


def all_shapes() -> list[tuple[str, Shape]]:
    return [(w.name, s) for w in WORKLOADS.values() for s in w.shapes]


def make_inputs(shape: Shape, seed: int | None = None):
    """Draw (q, k, v, rpb) on the CPU, in the workload dtype.

    Drawn in fp32 in the order q, k, v, rpb from one seeded generator, then
    rounded to the dtype.  Returns CPU tensors; q/k/v are [B, heads, H, W, D],
    rpb is [heads, 2k-1, 2k-1].
    """
    gen = torch.Generator(device="cpu")
    gen.manual_seed(shape.seed if seed is None else seed)
    dims = (shape.B, shape.heads, shape.H, shape.W, shape.D)
    q = torch.randn(dims, generator=gen, dtype=torch.float32)
    k = torch.randn(dims, generator=gen, dtype=torch.float32)
    v = torch.randn(dims, generator=gen, dtype=torch.float32)
    nb = 2 * shape.k - 1
    rpb = torch.randn((shape.heads, nb, nb), generator=gen, dtype=torch.float32) * 0.02
    dt = DTYPES[shape.dtype]
    return q.to(dt), k.to(dt), v.to(dt), rpb.to(dt)


def make_custom(B: int, heads: int, H: int, W: int, D: int, k: int, d: int, dtype: str, seed: int):
    """Inputs for an arbitrary shape (tests: ragged and edge cases)."""
    return make_inputs(Shape(B, heads, H, W, D, k, d, dtype, seed))
