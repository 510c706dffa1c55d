"""Seeded synthetic inputs for the Lighthouse Attention hot path.

This module only draws random tensors; it holds none of the method's
arithmetic. Both the CUDA path's tests/bench and the CPU oracle consume what
it returns, so it imports neither of them.

Workloads (named by what they are; shapes [B, N, H, D]):

  tiny_fp32   B1 H2  N1024   D64  fp32  p4 L3 K32    forward only, iid N(0,1)
  bf16_8k     B2 H8  N8192   D128 bf16  p4 L3 K256   iid N(0,1) times a per-token
              scale exp(U[ln 0.5, ln 2]) shared by Q, K, V and all heads
  ctx98k      B1 H16 N98304  D64  bf16  p4 L4 K512   iid N(0,1) (a 98K-context layer)
  ctx512k     B1 H16 N524288 D128 bf16  p8 L4 K1024  iid N(0,1); tokens with
              U(b,t) < 0.01 scaled x4 in Q, K, V, all heads (outlier norms)
  ties131k    B1 H8  N131072 D128 bf16  p4 L5 K512   per-head codebooks of 64 iid
              N(0,1) vectors for Q, K, V; one code per (b,t,h) shared by Q, K, V
              (many exactly tied scores); fixed-point accumulation mode

dO is iid N(0,1) for every workload. Draws are fp32 from torch's generator
seeded with (seed * 1000 + stream), streams Q=1 K=2 V=3 dO=4 scale=5
outlier=6 codebook=7 code-index=8; the fp32 draw is rounded to nearest-even
into the workload dtype. The stream on the CPU differs from the stream on a
CUDA device, so a test draws once and hands the same tensors to both sides.
"""

from __future__ import annotations

import math
from dataclasses import dataclass

import torch

__all__ = ["Workload", "WORKLOADS", "make_inputs", "make_dout", "torch_dtype"]


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    D: int
    dtype: str          # "fp32" | "bf16"
    p: int
    L: int
    K: int
    recipe: str         # "iid" | "token_scale" | "outliers" | "codebook"
    mode: str           # accumulation mode of the scatter steps: "fp" | "fixed"
    backward: bool
    seed: int


WORKLOADS = {
    w.name: w for w in [
        Workload("tiny_fp32", 1, 2, 1024, 64, "fp32", 4, 3, 32, "iid", "fp", False, 1),
        Workload("bf16_8k", 2, 8, 8192, 128, "bf16", 4, 3, 256, "token_scale", "fp", True, 2),
        Workload("ctx98k", 1, 16, 98304, 64, "bf16", 4, 4, 512, "iid", "fp", True, 3),
        Workload("ctx512k", 1, 16, 524288, 128, "bf16", 8, 4, 1024, "outliers", "fp", True, 4),
        Workload("ties131k", 1, 8, 131072, 128, "bf16", 4, 5, 512, "codebook", "fixed", True, 5),
        # the 512K inputs (same recipe and seed) with L = 1: the sub-sequence is the
        # whole token sequence, i.e. dense causal attention over all N tokens
        Workload("dense512k", 1, 16, 524288, 128, "bf16", 8, 1, 1024, "outliers", "fp", True, 4),
    ]
}


def torch_dtype(name: str) -> torch.dtype:
    return {"fp32": torch.float32, "bf16": torch.bfloat16}[name]


def _gen(seed: int, stream: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed * 1000 + stream)
    return g


def make_inputs(w: Workload, device="cpu", seed: int | None = None, N: int | None = None,
                B: int | None = None, H: int | None = None):
    """Draw (q, k, v) of shape [B, N, H, D] in the workload dtype on ``device``.

    ``N``/``B``/``H`` override the workload sizes (smaller cases of the same recipe).
    """
    seed = w.seed if seed is None else seed
    B = w.B if B is None else B
    N = w.N if N is None else N
    H = w.H if H is None else H
    D = w.D
    dt = torch_dtype(w.dtype)
    shape = (B, N, H, D)
    if w.recipe == "codebook":
        g7 = _gen(seed, 7, device)
        cq = torch.randn((H, 64, D), generator=g7, device=device)
        ck = torch.randn((H, 64, D), generator=g7, device=device)
        cv = torch.randn((H, 64, D), generator=g7, device=device)
        code = torch.randint(0, 64, (B, N, H), generator=_gen(seed, 8, device), device=device)
        hidx = torch.arange(H, device=device).view(1, 1, H).expand(B, N, H)
        out = [c[hidx, code].to(dt) for c in (cq, ck, cv)]
        return tuple(t.contiguous() for t in out)
    out = []
    for stream in (1, 2, 3):
        x = torch.randn(shape, generator=_gen(seed, stream, device), device=device)
        out.append(x)
    if w.recipe == "token_scale":
        u = torch.rand((B, N), generator=_gen(seed, 5, device), device=device)
        s = torch.exp(math.log(0.5) + u * (math.log(2.0) - math.log(0.5)))
        out = [x * s.view(B, N, 1, 1) for x in out]
    elif w.recipe == "outliers":
        u = torch.rand((B, N), generator=_gen(seed, 6, device), device=device)
        s = torch.where(u < 0.01, 4.0, 1.0)
        out = [x * s.view(B, N, 1, 1) for x in out]
    elif w.recipe != "iid":
        raise ValueError(w.recipe)
    return tuple(x.to(dt).contiguous() for x in out)


def make_dout(w: Workload, device="cpu", seed: int | None = None, N: int | None = None,
              B: int | None = None, H: int | None = None):
    """Draw the upstream gradient dO [B, N, H, D], iid N(0,1), in the workload dtype."""
    seed = w.seed if seed is None else seed
    B = w.B if B is None else B
    N = w.N if N is None else N
    H = w.H if H is None else H
    x = torch.randn((B, N, H, w.D), generator=_gen(seed, 4, device), device=device)
    return x.to(torch_dtype(w.dtype)).contiguous()
