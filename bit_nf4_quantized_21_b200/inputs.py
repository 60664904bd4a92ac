"""Seeded synthetic inputs for the QLoRA NF4 linear layer.

This module only draws random tensors and names workload shapes; it holds
none of the method's arithmetic, so both the CUDA path's tests and the CPU
oracle's tests can take their inputs from it.

Workloads (weights are nn.Linear-shaped [N = out, K = in], row-major):

  single   one 256x512 fp32 weight ~N(0, 0.02), seed 0; X 16x512 ~N(0,1);
           LoRA r=8, alpha=16, A, B ~N(0, 0.01); dY 16x256 ~N(0,1).
  llama7b  one LLaMA-7B-shaped layer: q/k/v/o 4096x4096, gate/up 11008x4096,
           down 4096x11008, bf16 ~N(0, 0.02); 2048 tokens (batch 4 x seq 512);
           r=16, alpha=32.
  decode   70B MLP shapes 28672x8192 and 8192x28672 ~N(0, 0.02) with 0.1% of
           the entries scaled x10 as outliers; M in {1, 4, 16}; r=16, alpha=32.
  stack7b  32 llama7b layers at 4096 tokens (batch 8 x seq 512).
  llama65b 80 layers of hidden 8192 / intermediate 22016 ~N(0, 0.015);
           8192 tokens; r=64, alpha=16.

Seeds: a matrix's seed is base*1000 + layer*7 + proj (proj order q, k, v, o,
gate, up, down; base = 0 single, 2 llama7b, 3 decode, 4 stack7b, 5 llama65b).
X, dY, A and B of a projection use seed*16 + 1, + 2, + 3, + 4.  Tensors are
drawn in fp32 and then cast to bf16 unless a workload says otherwise.  CPU
draws use torch's CPU generator; device draws use the CUDA (Philox)
generator, so the same seed gives different values on the two devices --
every comparison takes both sides' inputs from the same drawn tensor.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

PROJ_NAMES = ("q", "k", "v", "o", "gate", "up", "down")


def llama_shapes(hidden: int, inter: int) -> list[tuple[str, int, int]]:
    """(name, N, K) of the 7 projections of one decoder layer."""
    return [("q", hidden, hidden), ("k", hidden, hidden), ("v", hidden, hidden),
            ("o", hidden, hidden), ("gate", inter, hidden), ("up", inter, hidden),
            ("down", hidden, inter)]


@dataclass(frozen=True)
class Workload:
    name: str
    base_seed: int
    M: int
    r: int
    alpha: float
    w_std: float
    shapes: tuple = field(default_factory=tuple)   # ((name, N, K), ...)
    layers: int = 1
    w_dtype: str = "bf16"                          # dtype the weights are drawn in
    outlier_frac: float = 0.0
    outlier_scale: float = 10.0


SINGLE = Workload("single-256x512", 0, 16, 8, 16.0, 0.02, (("w", 256, 512),), 1, "f32")
LLAMA7B = Workload("llama7b-layer-m2048", 2, 2048, 16, 32.0, 0.02,
                   tuple(llama_shapes(4096, 11008)), 1)
DECODE = Workload("decode-70b-mlp", 3, 1, 16, 32.0, 0.02,
                  (("gate", 28672, 8192), ("down", 8192, 28672)), 1,
                  outlier_frac=1e-3, outlier_scale=10.0)
STACK7B = Workload("stack7b-32l-m4096", 4, 4096, 16, 32.0, 0.02,
                   tuple(llama_shapes(4096, 11008)), 32)
LLAMA65B = Workload("llama65b-80l-m8192", 5, 8192, 64, 16.0, 0.015,
                    tuple(llama_shapes(8192, 22016)), 80)

WORKLOADS = {w.name: w for w in (SINGLE, LLAMA7B, DECODE, STACK7B, LLAMA65B)}
DECODE_M = (1, 4, 16)


def matrix_seed(base: int, layer: int, proj: int) -> int:
    return base * 1000 + layer * 7 + proj


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def normal(shape, std: float, seed: int, device="cpu", dtype=torch.bfloat16) -> torch.Tensor:
    """~N(0, std^2) drawn in fp32, then cast to ``dtype``."""
    g = _gen(seed, device)
    t = torch.randn(tuple(shape), generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


def weight(shape, std: float, seed: int, device="cpu", dtype=torch.bfloat16,
           outlier_frac: float = 0.0, outlier_scale: float = 10.0) -> torch.Tensor:
    """A weight ~N(0, std^2); with ``outlier_frac`` > 0 a Bernoulli(outlier_frac)
    subset of the entries is multiplied by ``outlier_scale`` (before the cast)."""
    g = _gen(seed, device)
    t = torch.randn(tuple(shape), generator=g, device=device, dtype=torch.float32)
    t.mul_(std)
    if outlier_frac > 0.0:
        u = torch.rand(tuple(shape), generator=g, device=device, dtype=torch.float32)
        t = torch.where(u < outlier_frac, t * outlier_scale, t)
        del u
    return t.to(dtype)


def projection_inputs(wl: Workload, layer: int, proj: int, device="cpu", M: int | None = None,
                      with_weight: bool = True, with_grad: bool = True) -> dict:
    """All tensors of one projection: W (drawn dtype), X [M,K], dY [M,N],
    A [r,K], B [N,r] (bf16)."""
    name, N, K = wl.shapes[proj]
    M = wl.M if M is None else M
    s = matrix_seed(wl.base_seed, layer, proj)
    out = {"name": name, "N": N, "K": K, "M": M, "r": wl.r, "alpha": wl.alpha, "seed": s}
    if with_weight:
        wdt = torch.float32 if wl.w_dtype == "f32" else torch.bfloat16
        out["W"] = weight((N, K), wl.w_std, s, device, wdt, wl.outlier_frac, wl.outlier_scale)
    out["X"] = normal((M, K), 1.0, s * 16 + 1, device)
    if with_grad:
        out["dY"] = normal((M, N), 1.0, s * 16 + 2, device)
    out["A"] = normal((wl.r, K), 0.01, s * 16 + 3, device)
    out["B"] = normal((N, wl.r), 0.01, s * 16 + 4, device)
    return out
