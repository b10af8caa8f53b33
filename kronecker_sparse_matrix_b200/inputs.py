"""Seeded synthetic inputs for KS matrix products, shared by the tests, the smoke
check and the benchmark.

This module holds no KS arithmetic: it only draws random tensors and lists
patterns.  Both the CUDA path and the CPU oracle consume what it returns.

Recipe (the workloads of the KS-matmul abstract on the taxoreview.com page:
single factors shaped like ViT-S/16 and GPT-2-medium MLP projections, a
butterfly chain, and a sweep standing in for the abstract's "600 KS patterns",
whose list the pages do not give):

* one ``torch.Generator`` per workload, seeded as stated, on the device the
  tensors are made on; draw order is X first, then values (then the next
  factor's values for a chain);
* X ~ N(0, 1) unless stated (the toy uses U(-1, 1)); values ~ N(0, 1/c) (std
  1/sqrt(c)) unless stated (toy N(0, 1), butterfly N(0, 1/2));
* bf16 inputs are fp32 draws rounded to nearest-even bf16 (``Tensor.to``).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import List, Optional, Sequence, Tuple

import torch

Pattern = Tuple[int, int, int, int]

SWEEP_AD = (1, 2, 4, 8, 16, 32, 64)
SWEEP_BC = ((48, 48), (64, 64), (96, 96), (128, 128), (192, 192), (256, 256),
            (192, 48), (256, 64))
SWEEP_BATCH = 25088
SWEEP_MAX_WIDTH = 16384


def in_features(p: Pattern) -> int:
    a, b, c, d = p
    return a * c * d


def out_features(p: Pattern) -> int:
    a, b, c, d = p
    return a * b * d


def sweep_patterns() -> List[Pattern]:
    """The seeded sweep: a, d in {1,2,4,...,64}; (b, c) with both in
    {48,64,96,128,192,256} and b = c or b = 4c; a*b*d and a*c*d <= 16384.
    Literal reading of the set: 258 patterns, listed in a fixed order (the
    index is the pattern's seed)."""
    out = []
    for b, c in SWEEP_BC:
        for a in SWEEP_AD:
            for d in SWEEP_AD:
                if a * b * d <= SWEEP_MAX_WIDTH and a * c * d <= SWEEP_MAX_WIDTH:
                    out.append((a, b, c, d))
    return out


def butterfly_patterns(log2n: int = 12) -> List[Pattern]:
    """Square butterfly factors of size 2**log2n: (2^(k-1), 2, 2, 2^(log2n-k)),
    k = 1..log2n; the first entry is applied first."""
    return [(2 ** (k - 1), 2, 2, 2 ** (log2n - k)) for k in range(1, log2n + 1)]


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _cast(t: torch.Tensor, dtype: torch.dtype) -> torch.Tensor:
    return t if dtype == torch.float32 else t.to(dtype)


def draw_x(g: torch.Generator, batch: int, width: int, dist: str, device) -> torch.Tensor:
    if dist == "normal":
        return torch.randn(batch, width, generator=g, device=device, dtype=torch.float32)
    if dist == "uniform":  # U(-1, 1)
        u = torch.rand(batch, width, generator=g, device=device, dtype=torch.float32)
        return u.mul_(2.0).sub_(1.0)
    raise ValueError(dist)


def draw_values(g: torch.Generator, p: Pattern, std: float, device) -> torch.Tensor:
    a, b, c, d = p
    v = torch.randn(a, d, b, c, generator=g, device=device, dtype=torch.float32)
    return v.mul_(std) if std != 1.0 else v


@dataclass
class FactorInputs:
    pattern: Pattern
    batch: int
    X: torch.Tensor
    values: torch.Tensor
    dtype: torch.dtype


def factor_inputs(p: Pattern, batch: int, *, seed: int = 0, dtype=torch.float32,
                  device="cpu", x_dist: str = "normal",
                  v_std: Optional[float] = None) -> FactorInputs:
    """X (batch, a*c*d) then values [a][d][b][c], from one seeded generator."""
    a, b, c, d = p
    g = _gen(seed, device)
    X = draw_x(g, batch, a * c * d, x_dist, device)
    std = (1.0 / math.sqrt(c)) if v_std is None else float(v_std)
    V = draw_values(g, p, std, device)
    return FactorInputs(tuple(p), batch, _cast(X, dtype), _cast(V, dtype), dtype)


@dataclass
class ChainInputs:
    patterns: List[Pattern]
    batch: int
    X: torch.Tensor
    factors: List[torch.Tensor] = field(default_factory=list)
    dtype: torch.dtype = torch.float32


def chain_inputs(patterns: Sequence[Pattern], batch: int, *, seed: int = 0,
                 dtype=torch.float32, device="cpu", x_dist: str = "normal",
                 v_std: Optional[float] = None) -> ChainInputs:
    """X, then each factor's values in order, from one seeded generator."""
    g = _gen(seed, device)
    X = draw_x(g, batch, in_features(patterns[0]), x_dist, device)
    facs = []
    for p in patterns:
        std = (1.0 / math.sqrt(p[2])) if v_std is None else float(v_std)
        facs.append(_cast(draw_values(g, p, std, device), dtype))
    return ChainInputs([tuple(p) for p in patterns], batch, _cast(X, dtype), facs, dtype)


# Named workloads -----------------------------------------------------------

def toy(device="cpu") -> FactorInputs:
    """Pattern (2,4,4,2): K is 16x16 with 64 nonzeros; X 8x16 ~ U(-1,1);
    values ~ N(0,1); seed 0; fp32."""
    return factor_inputs((2, 4, 4, 2), 8, seed=0, device=device, x_dist="uniform", v_std=1.0)


VIT_PATTERN: Pattern = (1, 192, 48, 8)     # 384 -> 1536, ViT-S/16 MLP up-projection
VIT_BATCH = 25216                          # 128 images x 197 tokens
GPT2_PATTERN: Pattern = (1, 256, 64, 16)   # 1024 -> 4096, GPT-2-medium MLP up-projection
GPT2_BATCH = 8192                          # 8 x 1024 tokens
BUTTERFLY_LOG2N = 12
BUTTERFLY_BATCH = 4096


def vit(dtype=torch.float32, device="cpu", batch: int = VIT_BATCH, seed: int = 0) -> FactorInputs:
    return factor_inputs(VIT_PATTERN, batch, seed=seed, dtype=dtype, device=device)


def gpt2(dtype=torch.float32, device="cpu", batch: int = GPT2_BATCH, seed: int = 0) -> FactorInputs:
    return factor_inputs(GPT2_PATTERN, batch, seed=seed, dtype=dtype, device=device)


def butterfly(dtype=torch.float32, device="cpu", batch: int = BUTTERFLY_BATCH,
              log2n: int = BUTTERFLY_LOG2N, seed: int = 0) -> ChainInputs:
    return chain_inputs(butterfly_patterns(log2n), batch, seed=seed, dtype=dtype,
                        device=device, v_std=math.sqrt(0.5))


def sweep_inputs(index: int, dtype=torch.float32, device="cpu",
                 batch: int = SWEEP_BATCH) -> FactorInputs:
    """Sweep pattern number ``index`` with seed = index."""
    p = sweep_patterns()[index]
    return factor_inputs(p, batch, seed=index, dtype=dtype, device=device)
