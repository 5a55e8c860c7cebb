"""A seeded sweep of the calls' options against the FP64 oracle, three kinds of
case in turn: the cross-entropy pair on random rows (normal logits of several
widths, rows with +-80 outliers, confident rows whose target stands 10-60
above the rest, targets on outliers; ignore_index -100, -1, 7 or past V;
one gradient for every row or one per row; FP32, BF16 and in-place FP32
output), the vocabulary-parallel kernels on random, possibly empty, shard
splits, and the GEMMs' other outputs on integer operands (BF16 dW,
accumulated dW, and the direct-store epilogue of outputs a tensor map cannot
describe), which must be exact."""
import numpy as np
import pytest
import torch

import oracle
from helpers import assert_abs_close, assert_bf16_close, bits, guarded_empty, loss_tol, to_f64
from lm_head_fp32_b200 import lmhead, synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


def logits_case(rng, M, V):
    """Random FP32 logits [M,V] of one of four kinds, targets and an ignore_index."""
    kind = rng.integers(0, 4)
    x = rng.normal(0, float(rng.choice([0.5, 2.0, 4.0, 8.0])), size=(M, V)).astype(np.float32)
    if kind == 1:   # outliers
        for i in rng.choice(M, max(1, M // 10), replace=False):
            cols = rng.choice(V, min(V, 16), replace=False)
            x[i, cols] = rng.choice([-80.0, 80.0], size=len(cols))
    ign = int(rng.choice([-100, -1, 7, V + 5]))
    t = rng.integers(0, V, size=M).astype(np.int64)
    t[rng.random(M) < 0.1] = ign
    if kind == 2:   # confident rows
        gap = float(rng.choice([10.0, 30.0, 60.0]))
        x -= gap
        for i in range(M):
            if 0 <= t[i] < V:
                x[i, t[i]] = 2.0
    if kind == 3 and V > 1:  # targets on outliers
        for i in range(M):
            if 0 <= t[i] < V:
                x[i, t[i]] = float(rng.choice([-80.0, 80.0]))
    return torch.from_numpy(x), torch.from_numpy(t), ign


def ce_case(rng):
    """ce_fwd, then ce_bwd to FP32, to BF16 and in place, against the oracle."""
    M = int(rng.integers(1, 300))
    V = int(rng.integers(1, 9000))
    x, t, ign = logits_case(rng, M, V)
    xd, td = x.to(DEV), t.to(DEV)
    per_row = bool(rng.integers(0, 2))
    if per_row:
        g = torch.rand(M, generator=torch.Generator().manual_seed(int(rng.integers(1 << 30)))) + 0.5
    else:
        g = torch.tensor([float(rng.choice([1.0, 0.25, 3.0]))])
    st = guarded_empty((M, 4))
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    lmhead.ce_fwd(xd, td, st, ign, status)
    d32 = guarded_empty((M, V))
    d16 = guarded_empty((M, V), torch.bfloat16)
    gd = g.to(DEV)
    lmhead.ce_bwd(xd, td, st, gd, d32, ign, status)
    lmhead.ce_bwd(xd, td, st, gd, d16, ign, status)
    inplace = xd.clone()
    lmhead.ce_bwd(inplace, td, st, gd, inplace, ign, status)
    torch.cuda.synchronize()
    ref, code = oracle.ce_fwd(x.numpy(), t.numpy(), ign)
    valid = code == oracle.ROW_VALID
    got = st.cpu().double().numpy()
    assert np.array_equal(got[valid, 0], ref[valid, 0]) and np.array_equal(got[valid, 2], ref[valid, 2])
    assert_abs_close(got[valid, 1], ref[valid, 1], 1e-5 * ref[valid, 1], "d")
    assert_abs_close(got[:, 3], ref[:, 3], loss_tol(ref[:, 3]), "loss")
    gn = g.numpy().astype(np.float32)
    refd = oracle.ce_bwd(x.numpy(), t.numpy(), gn if per_row else float(gn[0]), ign)
    assert_abs_close(to_f64(d32), refd, 1e-6 * float(np.abs(gn).max()), "FP32 dlogits")
    assert_bf16_close(d16, refd, "BF16 dlogits")
    assert torch.equal(inplace, d32), "in-place"
    bad = ((t.numpy() != ign) & ((t.numpy() < 0) | (t.numpy() >= V))).any()
    assert (int(status.item()) & 1) == (1 if bad else 0)


def shard_case(rng):
    """The vocabulary split at random cuts (a shard may be empty and then
    contributes the neutral record): merged statistics and the shards'
    gradients against the oracle on the whole rows."""
    M = int(rng.integers(1, 200))
    V = int(rng.integers(8, 6000))
    x, t, ign = logits_case(rng, M, V)
    R = int(rng.integers(1, 5))
    cuts = sorted(set(int(c) for c in rng.integers(0, V + 1, size=R - 1)))
    bounds = [0] + cuts + [V]
    td = t.to(DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    recs, parts = [], []
    for a, b in zip(bounds[:-1], bounds[1:]):
        rec = guarded_empty((M, 4))
        if b > a:
            xr = x[:, a:b].contiguous().to(DEV)
            lmhead.ce_fwd_shard(xr, td, rec, a, V, ign, status)
            parts.append((a, b, xr))
        else:
            rec.copy_(torch.tensor([float("-inf"), 0.0, 0.0, 0.0], device=DEV).expand(M, 4))
        recs.append(rec)
    st = guarded_empty((M, 4))
    lmhead.ce_merge_shards(torch.stack(recs).contiguous(), td, st, V, ign, status)
    g = torch.tensor([1.0], device=DEV)
    dl = torch.zeros((M, V), device=DEV)
    for a, b, xr in parts:
        o = guarded_empty((M, b - a))
        lmhead.ce_bwd_shard(xr, td, st, g, o, a, V, ign, status)
        dl[:, a:b] = o
    torch.cuda.synchronize()
    ref, code = oracle.ce_fwd(x.numpy(), t.numpy(), ign)
    valid = code == oracle.ROW_VALID
    got = st.cpu().double().numpy()
    assert np.array_equal(got[valid, 0], ref[valid, 0]) and np.array_equal(got[valid, 2], ref[valid, 2])
    assert_abs_close(got[valid, 1], ref[valid, 1], 1e-5 * ref[valid, 1], "merged d")
    assert_abs_close(got[:, 3], ref[:, 3], loss_tol(ref[:, 3]), "merged loss")
    refd = oracle.ce_bwd(x.numpy(), t.numpy(), 1.0, ign)
    assert_abs_close(to_f64(dl), refd, 1e-6, "shard dlogits")


def gemm_case(rng):
    """Integer operands: BF16 dW, accumulated dW and the direct-store
    epilogue of all three GEMMs must equal the exact results."""
    M = int(rng.choice([1, 17, 64, 130, 257, 300, 700, 1100]))
    K = int(8 * rng.integers(1, 200))
    V = int(8 * rng.integers(1, max(2, min(5000, int(2e8 / (M * K))) // 8)))
    seed = int(rng.integers(1 << 20))
    dl = synth.int_bf16((M, V), seed)
    X = synth.int_bf16((M, K), seed + 1)
    W = synth.int_bf16((V, K), seed + 2)
    dld, Xd, Wd = dl.to(DEV), X.to(DEV), W.to(DEV)
    exact_w = oracle.dw(bits(dl), bits(X))
    exact_x = oracle.dx(bits(dl), bits(W))
    exact_l = oracle.logits(bits(X), bits(W))
    out16 = guarded_empty((V, K), torch.bfloat16)
    lmhead.lmhead_bwd_dw(dld, Xd, out16)
    dW0 = torch.randint(-500, 501, (V, K), generator=torch.Generator().manual_seed(seed)).float()
    acc = dW0.to(DEV).contiguous()
    lmhead.lmhead_bwd_dw_acc(dld, Xd, acc)
    # unaligned outputs take the direct-store epilogue
    def unaligned(shape, dt):
        n = shape[0] * shape[1]
        buf = torch.zeros(n + 8, dtype=dt, device=DEV)
        return buf, buf[1:1 + n].view(shape)
    bl, ul = unaligned((M, V), torch.float32)
    lmhead.lmhead_fwd(Xd, Wd, ul)
    bx, ux = unaligned((M, K), torch.float32)
    lmhead.lmhead_bwd_dx(dld, Wd, ux)
    bw, uw = unaligned((V, K), torch.float32)
    lmhead.lmhead_bwd_dw(dld, Xd, uw)
    torch.cuda.synchronize()
    assert np.array_equal(bits(out16), oracle.round_bf16(exact_w)), "dW BF16"
    assert torch.equal(acc.cpu(), dW0 + torch.from_numpy(exact_w).float()), "dW acc"
    assert np.array_equal(ul.cpu().numpy(), oracle.round_f32(exact_l)), "logits direct"
    assert np.array_equal(ux.cpu().numpy(), oracle.round_f32(exact_x)), "dX direct"
    assert np.array_equal(uw.cpu().numpy(), oracle.round_f32(exact_w)), "dW direct"
    for b, n in ((bl, M * V), (bx, M * K), (bw, V * K)):
        assert float(b[0]) == 0.0 and bool((b[1 + n:] == 0).all()), "wrote outside"


@pytest.mark.parametrize("case", range(30))
def test_option_sweep(case):
    rng = np.random.default_rng(20261203 + case)
    [ce_case, shard_case, gemm_case][case % 3](rng)
