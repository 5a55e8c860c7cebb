"""Seeded synthetic inputs for the LM-head loss path.

This module only draws random numbers and shapes them; it holds none of the
method's arithmetic.  Both the CUDA path (tests, bench) and the CPU oracle
consume its outputs, so the two sides always see identical bits.

Distributions and sizes follow the workloads the pages describe:
  * integer-valued BF16 operands uniform in [-8, 8] (both ends included),
    16 x K activations and 32768 x K vocabulary weights, seed 1234 --
    Megatron-LM PR #6252, "Integer bitwise exactness results" / "Method";
  * N = 32,768 vocabulary, M in {16, 128, 1024}, K in 1024..16384 for the
    FP32-versus-BF16 output sweep -- same page, "Tests" / "GEMM kernel
    benchmark";
  * rows of more than 100,000 columns for the cross-entropy kernels --
    TransformerEngine #2325, discussion of the saved m_d_X_y statistics.

Per-tensor seed streams: X = seed, W = seed+1, target = seed+2,
ignore mask = seed+3, outliers = seed+4.  ``torch.Generator`` on the CPU is
used for everything the oracle must reproduce at full size; a CUDA generator
(same seeds) is used only for the multi-GB cross-entropy inputs, whose sampled
rows are copied back to the host for the oracle.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import List, Optional, Tuple

import torch

IGNORE_INDEX = -100
SEED = 1234


def _gen(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def int_bf16(shape, seed: int, lo: int = -8, hi: int = 8, device="cpu") -> torch.Tensor:
    """BF16 tensor of integers drawn uniformly from [lo, hi] (inclusive); exact in BF16."""
    g = _gen(seed, device)
    t = torch.randint(lo, hi + 1, tuple(shape), generator=g, dtype=torch.int32, device=device)
    return t.to(torch.bfloat16)


def normal_bf16(shape, std: float, seed: int, device="cpu") -> torch.Tensor:
    """BF16 tensor drawn from N(0, std^2) (drawn in FP32, rounded RNE to BF16)."""
    g = _gen(seed, device)
    t = torch.randn(tuple(shape), generator=g, dtype=torch.float32, device=device)
    return (t * std).to(torch.bfloat16)


def ignore_rows(M: int, frac: float, seed: int) -> torch.Tensor:
    """Exactly floor(frac * M) distinct row indices from a seeded permutation."""
    n = int(math.floor(frac * M + 1e-9))
    if n == 0:
        return torch.empty(0, dtype=torch.int64)
    return torch.randperm(M, generator=_gen(seed))[:n].sort().values


def targets(M: int, V: int, ignore_frac: float, seed: int,
            ignore_index: int = IGNORE_INDEX) -> torch.Tensor:
    """int64 targets uniform in [0, V); floor(ignore_frac*M) rows set to ignore_index."""
    t = torch.randint(0, V, (M,), generator=_gen(seed + 2), dtype=torch.int64)
    rows = ignore_rows(M, ignore_frac, seed + 3)
    if rows.numel():
        t[rows] = ignore_index
    return t


def ce_logits(rows: int, cols: int, std: float, seed: int, outlier_frac: float = 0.0,
              outliers_per_row: int = 16, outlier_value: float = 80.0,
              device="cpu") -> Tuple[torch.Tensor, torch.Tensor]:
    """FP32 logits ~ N(0, std^2); in floor(outlier_frac*rows) rows, `outliers_per_row`
    distinct entries are replaced by +-outlier_value (sign 50/50).

    Returns (logits, outlier_rows)."""
    g = _gen(seed, device)
    x = torch.randn((rows, cols), generator=g, dtype=torch.float32, device=device)
    x.mul_(std)
    n = int(math.floor(outlier_frac * rows + 1e-9))
    orows = torch.empty(0, dtype=torch.int64)
    if n:
        go = _gen(seed + 4)
        orows = torch.randperm(rows, generator=go)[:n].sort().values
        for r in orows.tolist():
            c = torch.randperm(cols, generator=go)[:outliers_per_row]
            s = torch.randint(0, 2, (outliers_per_row,), generator=go).to(torch.float32) * 2 - 1
            x[r, c.to(device)] = (s * outlier_value).to(device)
    return x, orows


@dataclass
class GemmConfig:
    """One LM-head workload: X [M,K], W [V,K] (BF16), targets [M]."""
    name: str
    M: int
    K: int
    V: int
    dist: str                    # "int" (uniform integers in [-8,8]) or "normal"
    x_std: float = 1.0
    w_std: float = 0.02
    ignore_frac: float = 0.0
    grad: str = "inv_valid"       # "inv_valid" -> g = 1/num_valid, or "one"
    seed: int = SEED

    def make(self, device="cpu"):
        if self.dist == "int":
            X = int_bf16((self.M, self.K), self.seed, device=device)
            W = int_bf16((self.V, self.K), self.seed + 1, device=device)
        else:
            X = normal_bf16((self.M, self.K), self.x_std, self.seed, device=device)
            W = normal_bf16((self.V, self.K), self.w_std, self.seed + 1, device=device)
        t = targets(self.M, self.V, self.ignore_frac, self.seed)
        return X, W, t

    def grad_scalar(self, t: torch.Tensor) -> float:
        if self.grad == "one":
            return 1.0
        nv = int((t != IGNORE_INDEX).sum())
        return 1.0 / max(nv, 1)


@dataclass
class CEConfig:
    """Cross-entropy-only workload on FP32 rows."""
    name: str
    rows: int
    cols: int
    std: float
    outlier_frac: float
    ignore_frac: float
    outliers_per_row: int = 16
    outlier_value: float = 80.0
    seed: int = SEED

    def make(self, device="cpu"):
        x, orows = ce_logits(self.rows, self.cols, self.std, self.seed, self.outlier_frac,
                             self.outliers_per_row, self.outlier_value, device=device)
        t = targets(self.rows, self.cols, self.ignore_frac, self.seed)
        return x, t, orows


# The five workloads (sizes as the pages and the task fix them).
BITEXACT = GemmConfig("bitexact_16x512x32768", 16, 512, 32768, "int")
MIDSIZE = GemmConfig("lmhead_1024x4096x32768", 1024, 4096, 32768, "normal", ignore_frac=0.02)
LARGEVOCAB = GemmConfig("lmhead_4096x4096x128256", 4096, 4096, 128256, "normal", ignore_frac=0.01)
CE_WIDE = CEConfig("ce_8192x151936_outliers", 8192, 151936, 4.0, 0.01, 0.01)
SWEEP_M = (16, 128, 1024)
SWEEP_K = (1024, 2048, 4096, 8192, 16384)
SWEEP_V = 32768
EXACT_K = (512, 1024, 2048, 4096, 8192, 16384)


def sweep_configs() -> List[GemmConfig]:
    return [GemmConfig(f"sweep_M{m}_K{k}", m, k, SWEEP_V, "normal") for m in SWEEP_M for k in SWEEP_K]


def bf16_bits(t: torch.Tensor):
    """uint16 numpy view of a BF16 tensor's bit patterns (host copy)."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view("uint16")
