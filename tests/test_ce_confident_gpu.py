"""Rows whose target holds nearly all of the probability mass: the other
logits lie `gap` below the target's, so the loss runs from ~1 down to ~1e-23
and softmax_y - 1 cancels in FP32 (1/d - 1 with d = 1 + s).  The forward keeps
the other columns' share s apart from the target's term, the loss is
log1p(s exp(m - x_y)) and the backward takes the target's entry as
expm1(-loss) g, so on every path (ce_fwd, the fused forward, the
vocabulary-parallel shards) the loss holds the 1e-5 relative tolerance
without its absolute floor, the BF16 gradient is within 1 BF16 ulp of the
oracle's rounded value, and the FP32 gradient's target entry within 1e-5
relative.  The oracle computes the same quantities through s in FP64
(pinned against 60-digit decimal arithmetic)."""
import numpy as np
import pytest
import torch

import oracle
from lm_head_fp32_b200 import lmhead, synth
from helpers import assert_abs_close, assert_bf16_close, guarded_empty, to_f64

pytestmark = pytest.mark.gpu
DEV = "cuda"
GAPS = [0.0, 12.0, 30.0, 60.0]


def confident_logits(M, V, gap, seed):
    rng = np.random.default_rng(seed)
    x = (rng.normal(0, 1, size=(M, V)) - gap).astype(np.float32)
    t = rng.integers(0, V, size=M).astype(np.int64)
    t[::9] = -100
    for i in range(M):
        if t[i] >= 0:
            x[i, t[i]] = 2.5
    return torch.from_numpy(x), torch.from_numpy(t)


def check(stats, dl32, dl16, x, t, what):
    ref, code = oracle.ce_fwd(x.numpy(), t.numpy())
    valid = code == oracle.ROW_VALID
    got = stats.cpu().double().numpy()
    assert_abs_close(got[valid, 3], ref[valid, 3], 1e-5 * np.abs(ref[valid, 3]), f"{what}: loss")
    assert_abs_close(got[valid, 1], ref[valid, 1], 1e-5 * ref[valid, 1], f"{what}: d")
    refd = oracle.ce_bwd(x.numpy(), t.numpy(), 1.0)
    if dl16 is not None:
        assert_bf16_close(dl16, refd, f"{what}: BF16 dlogits")
    if dl32 is not None:
        d = to_f64(dl32)
        assert_abs_close(d, refd, 1e-6, f"{what}: FP32 dlogits")
        rows = np.nonzero(valid)[0]
        ty, ry = d[rows, t.numpy()[rows]], refd[rows, t.numpy()[rows]]
        assert_abs_close(ty, ry, 1e-5 * np.abs(ry), f"{what}: FP32 target entries")


@pytest.mark.parametrize("gap", GAPS)
@pytest.mark.parametrize("V", [4096, 4099])
def test_ce_fwd_bwd_confident_rows(gap, V):
    M = 48
    x, t = confident_logits(M, V, gap, 11 + int(gap) + V)
    xd, td = x.to(DEV), t.to(DEV)
    stats = guarded_empty((M, 4))
    dl32 = guarded_empty((M, V))
    dl16 = guarded_empty((M, V), torch.bfloat16)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    g = torch.ones(1, device=DEV)
    lmhead.ce_fwd(xd, td, stats, -100, status)
    lmhead.ce_bwd(xd, td, stats, g, dl32, -100, status)
    lmhead.ce_bwd(xd, td, stats, g, dl16, -100, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    check(stats, dl32, dl16, x, t, f"gap {gap}")


@pytest.mark.parametrize("gap", GAPS)
def test_fused_forward_confident_rows(gap):
    """The fused forward on confident rows: token i's activation row is the
    one-hot e_i and W[:, i] holds its wanted logits rounded to BF16, so the
    FP32 logits are exactly those values (one product 1 * value per entry)."""
    M, K, V = 40, 64, 2048
    x, t = confident_logits(M, V, gap, 21 + int(gap))
    # logits[i, v] = sum_k X[i,k] W[v,k] with X[i] = e_(i mod K) and W[v, k]
    # = the wanted logit of token k: exact when the wanted logits are BF16
    # values, so round them to BF16 first (the statistics then see exactly x)
    xb = x.to(torch.bfloat16)
    tok = torch.arange(M) % K
    X = torch.zeros((M, K), dtype=torch.bfloat16)
    X[torch.arange(M), tok] = 1.0
    W = torch.zeros((V, K), dtype=torch.bfloat16)
    W[:, tok] = xb.T
    logits = guarded_empty((M, V))
    stats = guarded_empty((M, 4))
    ws = guarded_empty((max(lmhead.lmhead_fwd_ce_workspace_bytes(M, V), 16),), torch.uint8)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    td = t.to(DEV)
    lmhead.lmhead_fwd_ce(X.to(DEV), W.to(DEV), td, logits, stats, ws, -100, status)
    dl16 = guarded_empty((M, V), torch.bfloat16)
    lmhead.ce_bwd(logits, td, stats, torch.ones(1, device=DEV), dl16, -100, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert torch.equal(logits.cpu(), xb.float())
    check(stats, None, dl16, xb.float(), t, f"fused, gap {gap}")


@pytest.mark.parametrize("gap", GAPS)
def test_vocabulary_shards_confident_rows(gap):
    """Three uneven shards: the shard holding the target leaves its term out
    of its record's sum, the merge adds it back."""
    M, bounds = 40, ((0, 700), (700, 356), (1056, 1000))
    V = sum(b[1] for b in bounds)
    x, t = confident_logits(M, V, gap, 31 + int(gap))
    td = t.to(DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    recs, parts = [], []
    for off, n in bounds:
        xr = x[:, off:off + n].contiguous().to(DEV)
        rec = guarded_empty((M, 4))
        lmhead.ce_fwd_shard(xr, td, rec, off, V, -100, status)
        recs.append(rec)
        parts.append(xr)
    stats = guarded_empty((M, 4))
    lmhead.ce_merge_shards(torch.stack(recs).contiguous(), td, stats, V, -100, status)
    dls = []
    for (off, n), xr in zip(bounds, parts):
        dl = guarded_empty((M, n))
        lmhead.ce_bwd_shard(xr, td, stats, torch.ones(1, device=DEV), dl, off, V, -100, status)
        dls.append(dl)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    check(stats, torch.cat(dls, dim=1), None, x, t, f"shards, gap {gap}")
