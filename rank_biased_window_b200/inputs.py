"""Seeded synthetic inputs for rank-factorised-bias attention.

This module holds no arithmetic of the method: it only draws random tensors.
Both the CUDA path and the fp64 oracle take their inputs from here, so the two
see the same bf16 bits.

Recipe (the same for every workload):
  * a torch CPU ``Generator`` seeded with ``SEED_BASE + workload index``;
  * draw order Q, K, V, U, W, then dO (only when a backward is needed);
  * Q, K, V, dO ~ N(0, 1); U, W ~ N(0, 1/r) (standard deviation r^-1/2);
  * every tensor drawn in fp32, then rounded to bf16 (round-to-nearest-even).

The workloads stand in for the pages' super-resolution settings: SwinIR-style
8x8 windows, PFT-style 32x32 windows ("Progressive Focused Transformer" notes,
key design section: 32x32 windows vs SwinIR's 8x8), attention over a whole
64x64 low-resolution feature map, and a 128x128 map, beyond the 96x96 windows
of "Rank-Factorized Implicit Neural Bias" (Abstract).  No dataset is used.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch

SEED_BASE = 20260306


@dataclass(frozen=True)
class Workload:
    name: str
    index: int
    B: int          # windows (or images) per call
    H: int          # heads
    N: int          # tokens per window
    d: int          # head dimension
    r: int          # bias rank
    backward: bool  # whether the workload includes the backward pass
    note: str

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def seed(self) -> int:
        return SEED_BASE + self.index

    def shape(self):
        return dict(B=self.B, H=self.H, N=self.N, d=self.d, r=self.r)


WORKLOADS = {
    "tiny": Workload("tiny", 0, 1, 1, 64, 32, 8, False,
                     "one 8x8 window, 1 head, d=32, r=8"),
    "swinir": Workload("swinir", 1, 1024, 6, 64, 32, 8, False,
                       "1024 SwinIR-style 8x8 windows, 6 heads, d=32, r=8"),
    "large": Workload("large", 2, 64, 6, 1024, 32, 16, False,
                      "64 windows of 32x32 tokens, 6 heads, d=32, r=16"),
    "global": Workload("global", 3, 4, 8, 4096, 64, 32, False,
                       "global attention over a 64x64 map, B=4, 8 heads, d=64, r=32"),
    "train": Workload("train", 4, 2, 8, 16384, 64, 32, True,
                      "training step fwd+bwd over a 128x128 map, B=2, 8 heads, d=64, r=32"),
}


def make_inputs(B: int, H: int, N: int, d: int, r: int, seed: int, *, with_dout: bool = False):
    """Return a dict of bf16 CPU tensors q, k, v, u, w (and dout).

    Shapes: q, k, v, dout ``[B, H, N, d]``; u, w ``[B, H, N, r]`` (r may be 0).
    """
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    out = {}
    for name in ("q", "k", "v"):
        out[name] = torch.randn((B, H, N, d), generator=g, dtype=torch.float32).to(torch.bfloat16)
    std = (1.0 / math.sqrt(r)) if r > 0 else 0.0
    for name in ("u", "w"):
        t = torch.randn((B, H, N, r), generator=g, dtype=torch.float32) * std
        out[name] = t.to(torch.bfloat16)
    if with_dout:
        out["dout"] = torch.randn((B, H, N, d), generator=g, dtype=torch.float32).to(torch.bfloat16)
    return out


def workload_inputs(w: Workload, *, with_dout: bool | None = None):
    wd = w.backward if with_dout is None else with_dout
    return make_inputs(w.B, w.H, w.N, w.d, w.r, w.seed, with_dout=wd)


def to_f64(t: torch.Tensor):
    """Exact bf16 -> float64 numpy conversion (every bf16 value is a double)."""
    return t.to(torch.float64).numpy()
