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

Out-of-bounds writes: every GPU output of the parity tests comes from
guarded_empty(), which places it between two 4 KiB guard bands filled with
0xFF bytes (a NaN in FP32 and in BF16, a value no kernel here writes); after
each GPU test the bands of every such buffer are checked (tests/conftest.py),
so a ragged tile or a partial vocabulary block that writes past its output is
caught even where the output's own values look right.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle


GUARD_BYTES = 4096
GUARD_FILL = 0xFF
_guarded = []


def guarded_empty(shape, dtype=torch.float32, device="cuda") -> torch.Tensor:
    """A contiguous output tensor with GUARD_BYTES of GUARD_FILL bytes just
    before and just after it (in the same allocation; the output stays
    16-byte aligned).  Its own contents are GUARD_FILL bytes too."""
    esize = torch.empty((), dtype=dtype).element_size()
    nb = GUARD_BYTES // esize
    n = math.prod(shape)
    raw = torch.empty(n + 2 * nb, dtype=dtype, device=device)
    raw.view(torch.uint8).fill_(GUARD_FILL)
    _guarded.append((raw, nb, n))
    return raw[nb:nb + n].view(tuple(shape))


def guarded_full(shape, value, dtype=torch.float32, device="cuda") -> torch.Tensor:
    t = guarded_empty(shape, dtype, device)
    t.fill_(value)
    return t


def check_guards():
    """Assert that no guard band of a buffer made since the last check was
    written, then forget those buffers."""
    if not _guarded:
        return
    torch.cuda.synchronize()
    bad = []
    for raw, nb, n in _guarded:
        b = raw.view(torch.uint8)
        esize = raw.element_size()
        for name, band in (("before", b[:nb * esize]), ("after", b[(nb + n) * esize:])):
            hit = torch.nonzero(band != GUARD_FILL).flatten()
            if hit.numel():
                bad.append(f"{tuple(raw.shape)} {raw.dtype}: {hit.numel()} bytes written {name} "
                           f"the output (first at band offset {int(hit[0])})")
    _guarded.clear()
    assert not bad, "; ".join(bad)


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


class FakeOps:
    """float64 restatement of the library calls' contracts, on CPU tensors."""

    @staticmethod
    def lmhead_fwd(X, W, out, status=None):
        out.copy_((X.double() @ W.double().T).float())

    @staticmethod
    def ce_fwd_shard(logits, target, rec, off, vtot, ignore, status=None):
        x = logits.double().numpy()
        V = x.shape[1]
        r = np.zeros((x.shape[0], 4))
        for i, y in enumerate(target.tolist()):
            if y == ignore or y < 0 or y >= vtot:
                continue
            m = x[i].max()
            own = off <= y < off + V
            e = np.exp(x[i] - m)
            # the shard that owns the target leaves its term out of the sum
            dx = np.delete(e, y - off).sum() if own else e.sum()
            r[i] = (m, dx, x[i, y - off] if own else 0.0, 1.0 if own else 0.0)
        rec.copy_(torch.from_numpy(r).float())

    @staticmethod
    def ce_merge_shards(recs, target, stats, vtot, ignore, status=None):
        R = recs.double().numpy()
        out = np.zeros((R.shape[1], 4))
        for i, y in enumerate(target.tolist()):
            if y == ignore or y < 0 or y >= vtot:
                continue
            m = R[:, i, 0].max()
            dx = (R[:, i, 1] * np.exp(R[:, i, 0] - m)).sum()   # every column but the target
            xy = R[R[:, i, 3] != 0, i, 2].sum()
            out[i] = (m, dx + np.exp(xy - m), xy, np.log1p(dx * np.exp(m - xy)))
        stats.copy_(torch.from_numpy(out).float())

    @staticmethod
    def ce_bwd_shard(logits, target, stats, g, dl, off, vtot, ignore, status=None):
        x = logits.double().numpy()
        st = stats.double().numpy()
        out = np.zeros_like(x)
        for i, y in enumerate(target.tolist()):
            if y == ignore or y < 0 or y >= vtot:
                continue
            out[i] = np.exp(x[i] - st[i, 0]) / st[i, 1]
            if off <= y < off + x.shape[1]:
                out[i, y - off] = np.expm1(-st[i, 3])   # softmax_y - 1 = exp(-loss) - 1
            out[i] *= float(g.reshape(-1)[0])
        dl.copy_(torch.from_numpy(out).to(dl.dtype))

    @staticmethod
    def lmhead_bwd_dx(dl, W, dX, status=None):
        dX.copy_((dl.double() @ W.double()).float())

    @staticmethod
    def lmhead_bwd_dw(dl, X, dW, status=None):
        dW.copy_((dl.double().T @ X.double()).float())
