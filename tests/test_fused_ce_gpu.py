"""Parity of lmhead_fwd_ce -- the vocabulary GEMM with the cross-entropy
forward statistics folded into its epilogue -- with the oracle and with the
separate lmhead_fwd + ce_fwd passes, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
from lm_head_fp32_b200 import lmhead, synth
from helpers import assert_abs_close, bits, guarded_empty, logits_tol, loss_tol

pytestmark = pytest.mark.gpu
DEV = "cuda"


def fused(X, W, t, ignore=-100):
    M, V = X.shape[0], W.shape[0]
    logits = guarded_empty((M, V), torch.float32)
    stats = guarded_empty((M, 4), torch.float32)
    ws = guarded_empty((max(lmhead.lmhead_fwd_ce_workspace_bytes(M, V), 16),), torch.uint8,
                     device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    lmhead.lmhead_fwd_ce(X.to(DEV), W.to(DEV), t.to(DEV), logits, stats, ws, ignore, status)
    torch.cuda.synchronize()
    return logits, stats, int(status.item())


def separate(X, W, t, ignore=-100):
    M, V = X.shape[0], W.shape[0]
    logits = guarded_empty((M, V), torch.float32)
    stats = guarded_empty((M, 4), torch.float32)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    lmhead.lmhead_fwd(X.to(DEV), W.to(DEV), logits, status)
    lmhead.ce_fwd(logits, t.to(DEV), stats, ignore, status)
    torch.cuda.synchronize()
    return logits, stats, int(status.item())


def check(X, W, t, ignore=-100, rows=None):
    lf, sf, stf = fused(X, W, t, ignore)
    ls, ss, sts = separate(X, W, t, ignore)
    assert stf == sts
    assert torch.equal(lf, ls), "fused logits differ from lmhead_fwd's"
    lg = lf.cpu().numpy() if rows is None else lf[torch.as_tensor(rows, device=DEV)].cpu().numpy()
    tt = t.numpy() if rows is None else t.numpy()[rows]
    ref, code = oracle.ce_fwd(lg, tt, ignore)
    got = (sf if rows is None else sf[torch.as_tensor(rows, device=DEV)]).cpu().double().numpy()
    valid = code == oracle.ROW_VALID
    assert np.array_equal(got[valid, 0], ref[valid, 0]), "row max"
    assert np.array_equal(got[valid, 2], ref[valid, 2]), "target logit"
    assert_abs_close(got[valid, 1], ref[valid, 1], 1e-5 * ref[valid, 1], "sum-exp d")
    assert_abs_close(got[:, 3], ref[:, 3], loss_tol(ref[:, 3]), "loss")
    assert (got[~valid] == 0).all()
    # and against the separate ce_fwd kernel (same math, other merge order)
    other = (ss if rows is None else ss[torch.as_tensor(rows, device=DEV)]).cpu().double().numpy()
    assert_abs_close(got[:, 3], other[:, 3], 2 * loss_tol(other[:, 3]), "loss vs ce_fwd")
    return lf, sf


@pytest.mark.parametrize("M,K,V", [(16, 512, 32768), (300, 264, 1000), (17, 72, 32776),
                                   (130, 1024, 520), (257, 136, 2052), (1, 8, 4),
                                   (64, 4096, 128256), (128, 1024, 8200),
                                   (300, 136, 200), (140, 256, 252), (96, 16384, 520)])
def test_fused_ce_matches_oracle(M, K, V):
    X = synth.normal_bf16((M, K), 1.0, 51 + M)
    W = synth.normal_bf16((V, K), 0.05, 52 + V)
    t = synth.targets(M, V, 0.1, 53 + M)
    rows = None if M * V <= 4_000_000 else np.arange(0, M, 7)
    check(X, W, t, rows=rows)


def test_fused_ce_integer_inputs_bit_exact_logits():
    cfg = synth.BITEXACT
    X, W, t = cfg.make()
    lf, sf = check(X, W, t)
    ref = oracle.round_f32(oracle.logits(bits(X), bits(W)))
    assert np.array_equal(lf.cpu().numpy().view(np.uint32), ref.view(np.uint32))


def test_fused_ce_bad_targets_and_custom_ignore_index():
    M, K, V = 40, 128, 4096
    X = synth.normal_bf16((M, K), 1.0, 61)
    W = synth.normal_bf16((V, K), 0.05, 62)
    t = synth.targets(M, V, 0.0, 63)
    t[3] = V          # out of range
    t[5] = -1         # out of range
    t[7] = 11         # the ignore_index of this call
    t[9] = 11
    lf, sf, status = fused(X, W, t, ignore=11)
    assert status & lmhead.DEV_BAD_TARGET
    for r in (3, 5, 7, 9):
        assert (sf[r] == 0).all()
    check(X, W, t, ignore=11)


def test_fused_ce_every_row_ignored():
    """Every target is ignore_index: the logits are still those of lmhead_fwd,
    every statistics row is zero and no status bit is set."""
    M, K, V = 40, 256, 1000
    X = synth.normal_bf16((M, K), 1.0, 5)
    W = synth.normal_bf16((V, K), 0.02, 6)
    t = torch.full((M,), -100, dtype=torch.int64)
    lf, sf, st = fused(X, W, t)
    ls, _, _ = separate(X, W, t)
    assert st == 0
    assert torch.equal(lf, ls)
    assert (sf == 0).all()


def test_fused_ce_fallback_paths():
    # V % 4 != 0: the logits cannot go through the TMA-store epilogue, so the call
    # runs the two separate passes; the results still match the oracle
    M, K, V = 33, 64, 1001
    X = synth.normal_bf16((M, K), 1.0, 71)
    W = synth.normal_bf16((V, K), 0.05, 72)
    t = synth.targets(M, V, 0.1, 73)
    check(X, W, t)


def test_fused_ce_deterministic_and_midsize_config():
    cfg = synth.MIDSIZE
    X, W, t = cfg.make()
    a = fused(X, W, t)
    b = fused(X, W, t)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
    assert a[2] == 0
    check(X, W, t, rows=np.arange(0, cfg.M, 5))
