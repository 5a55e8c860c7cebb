"""A seeded sweep of random shapes through all five calls and the fused
forward, against the FP64 oracle.  The shapes are drawn so that together they
reach every GEMM variant the library picks by size: token tiles of 16, 32,
64, 128 and 256 (single CTA, two CTAs per SM, and CTA pairs), ragged m, n and
k tails, dX tiles split into two parts (a sparse last wave) and unsplit, FP32
and BF16 outputs.  Half of the cases use integer operands, for which every
GEMM output must equal the oracle word for word."""
import numpy as np
import pytest
import torch

import oracle
from lm_head_fp32_b200 import lmhead, synth
from helpers import (assert_abs_close, assert_bf16_close, bits, gemm_tol, guarded_empty,
                     logits_tol, loss_tol, to_f64)

pytestmark = pytest.mark.gpu
DEV = "cuda"
BUDGET = 4e8          # multiply-adds per GEMM, so the oracle stays within seconds


def _shapes(n=16, seed=20261203):
    rng = np.random.default_rng(seed)
    tokens = [1, 9, 16, 23, 32, 47, 64, 100, 128, 129, 200, 256, 300, 511, 640, 1100]
    out = []
    for i in range(n):
        M = int(tokens[i % len(tokens)])
        K = int(8 * rng.integers(1, 160))                   # 8 .. 1272
        vmax = max(8, int(BUDGET / (M * K)) // 8 * 8)
        V = int(8 * rng.integers(1, max(2, min(vmax, 40000) // 8)))
        out.append((M, K, V, bool(i % 2)))
    return out


@pytest.mark.parametrize("M,K,V,integer", _shapes())
def test_random_shape_through_the_path(M, K, V, integer):
    seed = 7 * M + 3 * K + V
    if integer:
        X, W = synth.int_bf16((M, K), seed), synth.int_bf16((V, K), seed + 1)
        dl = synth.int_bf16((M, V), seed + 2)            # integer "dlogits" for exact GEMMs
    else:
        X = synth.normal_bf16((M, K), 1.0, seed)
        W = synth.normal_bf16((V, K), 0.05, seed + 1)
        dl = synth.normal_bf16((M, V), 1e-3, seed + 2)
    t = synth.targets(M, V, 0.1, seed)
    Xd, Wd, dld, td = X.to(DEV), W.to(DEV), dl.to(DEV), t.to(DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    logits = guarded_empty((M, V))
    logits16 = guarded_empty((M, V), torch.bfloat16)
    lmhead.lmhead_fwd(Xd, Wd, logits, st)
    lmhead.lmhead_fwd(Xd, Wd, logits16, st)
    stats = guarded_empty((M, 4))
    lmhead.ce_fwd(logits, td, stats, -100, st)
    g = torch.tensor([0.5], device=DEV)
    dlog = guarded_empty((M, V), torch.bfloat16)
    lmhead.ce_bwd(logits, td, stats, g, dlog, -100, st)
    dX, dW = guarded_empty((M, K)), guarded_empty((V, K))
    dX16 = guarded_empty((M, K), torch.bfloat16)
    lmhead.lmhead_bwd_dx(dld, Wd, dX, st)
    lmhead.lmhead_bwd_dx(dld, Wd, dX16, st)
    lmhead.lmhead_bwd_dw(dld, Xd, dW, st)
    fl = guarded_empty((M, V))
    fs = guarded_empty((M, 4))
    ws = guarded_empty((max(lmhead.lmhead_fwd_ce_workspace_bytes(M, V), 16),), torch.uint8)
    lmhead.lmhead_fwd_ce(Xd, Wd, td, fl, fs, ws, -100, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0

    ref_l = oracle.logits(bits(X), bits(W))
    ref_dx = oracle.dx(bits(dl), bits(W))
    ref_dw = oracle.dw(bits(dl), bits(X))
    if integer:
        assert np.array_equal(logits.cpu().numpy(), oracle.round_f32(ref_l))
        assert np.array_equal(bits(logits16), oracle.round_bf16(ref_l))
        assert np.array_equal(dX.cpu().numpy(), oracle.round_f32(ref_dx))
        assert np.array_equal(dW.cpu().numpy(), oracle.round_f32(ref_dw))
    else:
        assert_abs_close(to_f64(logits), ref_l, logits_tol(X, W), "logits")
        assert_bf16_close(logits16, ref_l, "BF16 logits", abs_tol=logits_tol(X, W))
        assert_abs_close(to_f64(dX), ref_dx, gemm_tol(V, dl, W), "dX")
        assert_abs_close(to_f64(dW), ref_dw, gemm_tol(M, dl, X), "dW")
    assert_bf16_close(dX16, ref_dx, "BF16 dX", abs_tol=gemm_tol(V, dl, W))
    # the cross-entropy stages on the GPU's logits
    lg = logits.cpu().numpy()
    ref_s, code = oracle.ce_fwd(lg, t.numpy())
    got = stats.cpu().double().numpy()
    valid = code == oracle.ROW_VALID
    assert np.array_equal(got[valid, 0], ref_s[valid, 0]) and np.array_equal(got[valid, 2], ref_s[valid, 2])
    assert_abs_close(got[:, 3], ref_s[:, 3], loss_tol(ref_s[:, 3]), "loss")
    assert_bf16_close(dlog, oracle.ce_bwd(lg, t.numpy(), 0.5), "BF16 dlogits")
    # the fused forward: the same logits, statistics within the CE tolerances
    assert torch.equal(fl, logits)
    fg = fs.cpu().double().numpy()
    assert np.array_equal(fg[valid, 0], got[valid, 0]) and np.array_equal(fg[valid, 2], got[valid, 2])
    assert_abs_close(fg[:, 3], ref_s[:, 3], loss_tol(ref_s[:, 3]), "fused loss")
