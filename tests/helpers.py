"""Comparison helpers shared by the parity tests (no method arithmetic here).

Tolerances, from the contract the tests enforce:
  * integer-valued inputs: bit-exact;
  * FP32 logits: |gpu - oracle| <= 1e-5 * sqrt(K) * max|x| * max|w|;
  * per-row loss: |gpu - oracle| <= 1e-5 * |oracle| + 1e-6 (absolute floor for
    a loss near zero);
  * FP32 dlogits: |gpu - oracle| <= 1e-6;
  * every BF16 output: within one BF16 ulp of the oracle value rounded to BF16
    (RNE), a GPU zero accepted where |oracle| < 2^-126 (flush to zero).  A
    GEMM's BF16 output is the rounding of its FP32 accumulator, which may
    already differ from the exact value by the FP32 tolerance; near
    cancellation that exceeds one BF16 ulp of the tiny result, so for GEMM
    outputs the bound is one ulp plus the FP32 tolerance (abs_tol);
  * dX / dW on random inputs: 1e-5 * sqrt(reduction length) * max|a| * max|b|.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().double().numpy() if t.dtype == torch.bfloat16 \
        else t.detach().cpu().double().numpy()


def bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def bf16_ulp(a: np.ndarray) -> np.ndarray:
    """Spacing of BF16 numbers at |a| (8 significant bits; subnormal step 2^-133)."""
    a = np.abs(np.asarray(a, dtype=np.float64))
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, -126.0)
    return np.exp2(e - 7.0)


def assert_bf16_close(gpu_bf16: torch.Tensor, ref_f64: np.ndarray, what: str, abs_tol=0.0):
    """|gpu - RNE_bf16(ref)| <= 1 ulp of BF16 at max(|gpu|, |ref|) (+ abs_tol)."""
    g = to_f64(gpu_bf16)
    r = oracle.bf16_bits_to_f64(oracle.round_bf16(ref_f64))
    ulp = bf16_ulp(np.maximum(np.abs(g), np.abs(r)))
    ftz = (g == 0) & (np.abs(ref_f64) < 2.0 ** -126)
    bad = (np.abs(g - r) > ulp + abs_tol) & ~ftz
    if bad.any():
        idx = np.argwhere(bad)[:5]
        raise AssertionError(f"{what}: {int(bad.sum())} BF16 elements off by more than 1 ulp; "
                             f"first {idx.tolist()}: gpu {g[bad][:5]} ref {r[bad][:5]}")


def assert_abs_close(gpu: np.ndarray, ref: np.ndarray, tol, what: str):
    d = np.abs(np.asarray(gpu, np.float64) - np.asarray(ref, np.float64))
    tol = np.broadcast_to(np.asarray(tol, np.float64), d.shape)
    bad = ~(d <= tol)
    if bad.any():
        i = np.argwhere(bad)[:5]
        raise AssertionError(f"{what}: {int(bad.sum())} elements beyond tolerance; worst "
                             f"|diff| {float(np.nanmax(d)):.3e} (tol {float(tol.flat[0]):.3e}); "
                             f"first {i.tolist()}")


def logits_tol(X: torch.Tensor, W: torch.Tensor) -> float:
    K = X.shape[1]
    return 1e-5 * math.sqrt(K) * float(X.float().abs().max()) * float(W.float().abs().max())


def gemm_tol(red_len: int, a: torch.Tensor, b: torch.Tensor) -> float:
    return 1e-5 * math.sqrt(red_len) * float(a.float().abs().max()) * float(b.float().abs().max())


def loss_tol(ref: np.ndarray) -> np.ndarray:
    return 1e-5 * np.abs(ref) + 1e-6
