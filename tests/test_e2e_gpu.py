"""The whole path (lmhead_fwd -> ce_fwd -> ce_bwd -> lmhead_bwd_dx ->
lmhead_bwd_dw) on the three LM-head workloads, each stage compared with the
oracle fed the GPU's own inputs to that stage (so an error is caught at the
stage that makes it).  Full comparison where the oracle finishes in seconds,
sampled rows otherwise."""
import numpy as np
import pytest
import torch

import oracle
from lm_head_fp32_b200 import lmhead, synth
from helpers import (assert_abs_close, assert_bf16_close, bits, gemm_tol, guarded_empty,
                     logits_tol, loss_tol, to_f64)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def run_path(cfg):
    X, W, t = cfg.make()
    M, K, V = cfg.M, cfg.K, cfg.V
    g = cfg.grad_scalar(t)
    Xd, Wd, td = X.to(DEV), W.to(DEV), t.to(DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    logits = guarded_empty((M, V), torch.float32)
    stats = guarded_empty((M, 4), torch.float32)
    dl = guarded_empty((M, V), torch.bfloat16)
    dX = guarded_empty((M, K), torch.float32)
    dW = guarded_empty((V, K), torch.float32)
    gd = torch.tensor([g], dtype=torch.float32, device=DEV)
    lmhead.lmhead_fwd(Xd, Wd, logits, status)
    lmhead.ce_fwd(logits, td, stats, -100, status)
    lmhead.ce_bwd(logits, td, stats, gd, dl, -100, status)
    lmhead.lmhead_bwd_dx(dl, Wd, dX, status)
    lmhead.lmhead_bwd_dw(dl, Xd, dW, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return dict(X=X, W=W, t=t, g=g, logits=logits, stats=stats, dl=dl, dX=dX, dW=dW)


def check(cfg, r, token_rows, vocab_rows, exact_logits=False):
    X, W, t, g = r["X"], r["W"], r["t"], r["g"]
    xb, wb = bits(X), bits(W)
    tr = torch.as_tensor(token_rows, device=DEV)
    # a1 logits
    ref_l = oracle.logits(xb, wb, rows=token_rows)
    got_l = r["logits"][tr].cpu().numpy()
    if exact_logits:
        assert np.array_equal(got_l.view(np.uint32), oracle.round_f32(ref_l).view(np.uint32))
    else:
        assert_abs_close(got_l, ref_l, logits_tol(X, W), "logits")
    # a2 / a3 on the GPU's logits of those rows
    lg = r["logits"][tr].cpu().numpy()
    tt = t.numpy()[token_rows]
    st_ref, code = oracle.ce_fwd(lg, tt)
    st = r["stats"][tr].cpu().double().numpy()
    assert_abs_close(st[:, 3], st_ref[:, 3], loss_tol(st_ref[:, 3]), "loss")
    assert (st[code != oracle.ROW_VALID] == 0).all()
    dl_ref = oracle.ce_bwd(lg, tt, g)
    assert_bf16_close(r["dl"][tr], dl_ref, "BF16 dlogits")
    # a4 / a5 on the GPU's BF16 dlogits
    dlb = bits(r["dl"])
    assert_abs_close(to_f64(r["dX"][tr]), oracle.dx(dlb, wb, rows=token_rows),
                     gemm_tol(cfg.V, r["dl"], W), "dX")
    assert_abs_close(to_f64(r["dW"][torch.as_tensor(vocab_rows, device=DEV)]),
                     oracle.dw(dlb, xb, vrows=vocab_rows), gemm_tol(cfg.M, r["dl"], X), "dW")
    for k in ("logits", "stats", "dl", "dX", "dW"):
        assert bool(torch.isfinite(r[k]).all()), k


def test_bitexact_smoke_config_full():
    cfg = synth.BITEXACT
    r = run_path(cfg)
    check(cfg, r, np.arange(cfg.M), np.arange(0, cfg.V, 97), exact_logits=True)


def test_midsize_config_sampled():
    cfg = synth.MIDSIZE
    r = run_path(cfg)
    rng = np.random.default_rng(cfg.seed + 5)
    ign = np.nonzero(r["t"].numpy() == -100)[0][:4]
    rows = np.unique(np.concatenate([rng.choice(cfg.M, 20, replace=False), ign, [cfg.M - 1]]))
    vrows = np.unique(np.concatenate([rng.choice(cfg.V, 40, replace=False), [0, cfg.V - 1]]))
    check(cfg, r, rows, vrows)
    # the CE stages on every row: loss and BF16 dlogits over the full batch
    lg = r["logits"].cpu().numpy()
    st_ref, _ = oracle.ce_fwd(lg, r["t"].numpy())
    st = r["stats"].cpu().double().numpy()
    assert_abs_close(st[:, 3], st_ref[:, 3], loss_tol(st_ref[:, 3]), "loss (all rows)")


def test_large_vocab_config_sampled():
    cfg = synth.LARGEVOCAB
    r = run_path(cfg)
    rng = np.random.default_rng(cfg.seed + 5)
    ign = np.nonzero(r["t"].numpy() == -100)[0][:2]
    # rows from 3328 on are the last wave of dX's tiles, computed in two k-halves
    rows = np.unique(np.concatenate([rng.choice(cfg.M, 6, replace=False), ign,
                                     [3328, 3711, cfg.M - 1]]))
    vrows = np.unique(np.concatenate([rng.choice(cfg.V, 12, replace=False), [cfg.V - 1]]))
    check(cfg, r, rows, vrows)
