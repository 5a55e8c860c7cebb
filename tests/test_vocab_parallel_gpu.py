"""Vocabulary-parallel cross-entropy kernels on one GPU: the vocabulary is
split into uneven shards, each shard's part runs through the C ABI
(ce_fwd_shard, ce_merge_shards, ce_bwd_shard, and the GEMMs on the shard), and
the results are checked against the oracle on the whole vocabulary and
against the single-device calls.  No rank waits on another: the shards' calls
simply run one after the other on one stream."""
import numpy as np
import pytest
import torch

import oracle
from lm_head_fp32_b200 import lmhead, synth, vocab_parallel
from helpers import assert_abs_close, assert_bf16_close, bits, gemm_tol, guarded_empty, loss_tol, to_f64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _case(M=96, K=128, bounds=((0, 400), (400, 344), (744, 256)), seed=7):
    V = sum(b[1] for b in bounds)
    X = synth.normal_bf16((M, K), 1.0, seed)
    W = synth.normal_bf16((V, K), 0.1, seed + 1)
    t = synth.targets(M, V, 0.05, seed)
    t[1] = V + 3          # a bad target
    return X, W, t, V, bounds


def test_shards_match_whole_vocabulary():
    X, W, t, V, bounds = _case()
    M, K = X.shape
    Xd, td = X.to(DEV), t.to(DEV)
    g = torch.tensor([0.5], device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    recs, logits = [], []
    for off, n in bounds:
        Wr = W[off:off + n].contiguous().to(DEV)
        lr = guarded_empty((M, n))
        lmhead.lmhead_fwd(Xd, Wr, lr, status)
        rec = guarded_empty((M, 4))
        lmhead.ce_fwd_shard(lr, td, rec, off, V, -100, status)
        recs.append(rec)
        logits.append(lr)
    stats = guarded_empty((M, 4))
    lmhead.ce_merge_shards(torch.stack(recs).contiguous(), td, stats, V, -100, status)
    dls = []
    for (off, n), lr in zip(bounds, logits):
        dl = guarded_empty((M, n), torch.bfloat16)
        lmhead.ce_bwd_shard(lr, td, stats, g, dl, off, V, -100, status)
        dls.append(dl)
    torch.cuda.synchronize()
    assert int(status.item()) == lmhead.DEV_BAD_TARGET      # only the planted bad target
    full = torch.cat(logits, dim=1)
    # whole-vocabulary statistics against the oracle on the same logits
    ref, code = oracle.ce_fwd(full.cpu().numpy(), t.numpy())
    got = stats.cpu().double().numpy()
    valid = code == oracle.ROW_VALID
    assert np.array_equal(got[valid, 0], ref[valid, 0]) and np.array_equal(got[valid, 2], ref[valid, 2])
    assert_abs_close(got[:, 3], ref[:, 3], loss_tol(ref[:, 3]), "merged loss")
    assert (got[~valid] == 0).all()
    # and against the single-device ce_fwd
    one = guarded_empty((M, 4))
    lmhead.ce_fwd(full.contiguous(), td, one, -100)
    torch.cuda.synchronize()
    assert_abs_close(got[:, 3], one.cpu().double().numpy()[:, 3], 2 * loss_tol(ref[:, 3]), "vs ce_fwd")
    # gradients on the shards = gradient of the whole row
    dl_full = torch.cat(dls, dim=1)
    assert_bf16_close(dl_full, oracle.ce_bwd(full.cpu().numpy(), t.numpy(), 0.5), "shard dlogits")
    # dX = sum over shards, dW = per-shard rows
    dX = torch.zeros((M, K), device=DEV)
    for (off, n), dl in zip(bounds, dls):
        part = guarded_empty((M, K))
        lmhead.lmhead_bwd_dx(dl, W[off:off + n].contiguous().to(DEV), part)
        dX += part
    dlb = bits(dl_full)
    assert_abs_close(to_f64(dX), oracle.dx(dlb, bits(W)), gemm_tol(V, dl_full, W), "dX")


def test_step_on_one_device_equals_five_calls():
    X, W, t, V, _ = _case(M=64, K=64, bounds=((0, 512),), seed=11)
    Xd, Wd, td = X.to(DEV), W.to(DEV), t.to(DEV)
    g = torch.tensor([0.25], device=DEV)
    stats, dX, dW, logits, dl = vocab_parallel.step(Xd, Wd, td, 0, V, g)
    M, K = X.shape
    ref_l = guarded_empty((M, V))
    lmhead.lmhead_fwd(Xd, Wd, ref_l)
    ref_s = guarded_empty((M, 4))
    lmhead.ce_fwd(ref_l, td, ref_s)
    ref_dl = guarded_empty((M, V), torch.bfloat16)
    lmhead.ce_bwd(ref_l, td, ref_s, g, ref_dl)
    torch.cuda.synchronize()
    assert torch.equal(logits, ref_l)
    # one shard: the merge is the identity on (m, d) and recomputes the loss
    assert torch.equal(stats[:, :3], ref_s[:, :3])
    assert_abs_close(stats[:, 3].cpu().numpy(), ref_s[:, 3].cpu().numpy(),
                     loss_tol(ref_s[:, 3].cpu().double().numpy()), "loss")
    assert torch.equal(dl, ref_dl)
    ref_dx = torch.empty_like(dX)
    lmhead.lmhead_bwd_dx(ref_dl, Wd, ref_dx)
    ref_dw = torch.empty_like(dW)
    lmhead.lmhead_bwd_dw(ref_dl, Xd, ref_dw)
    torch.cuda.synchronize()
    assert torch.equal(dX, ref_dx) and torch.equal(dW, ref_dw)


def test_merge_with_an_empty_shard_record():
    """A rank whose vocabulary shard is empty contributes the neutral record
    {-inf, 0, 0, 0} (vocab_parallel.step); merging it with the other shards'
    records must give the same statistics as merging those alone."""
    X, W, t, V, bounds = _case(M=40, K=64, bounds=((0, 200), (200, 144)), seed=13)
    M = X.shape[0]
    Xd, td = X.to(DEV), t.to(DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    recs = []
    for off, n in bounds:
        lr = guarded_empty((M, n))
        lmhead.lmhead_fwd(Xd, W[off:off + n].contiguous().to(DEV), lr, status)
        rec = guarded_empty((M, 4))
        lmhead.ce_fwd_shard(lr, td, rec, off, V, -100, status)
        recs.append(rec)
    empty = torch.zeros((M, 4), device=DEV)
    empty[:, 0] = float("-inf")
    with_empty = guarded_empty((M, 4))
    lmhead.ce_merge_shards(torch.stack(recs + [empty]).contiguous(), td, with_empty, V, -100, status)
    first_empty = guarded_empty((M, 4))
    lmhead.ce_merge_shards(torch.stack([empty] + recs).contiguous(), td, first_empty, V, -100, status)
    without = guarded_empty((M, 4))
    lmhead.ce_merge_shards(torch.stack(recs).contiguous(), td, without, V, -100, status)
    torch.cuda.synchronize()
    assert int(status.item()) == lmhead.DEV_BAD_TARGET      # only the planted bad target
    assert torch.equal(with_empty, without) and torch.equal(first_empty, without)
    assert bool(torch.isfinite(without).all())
