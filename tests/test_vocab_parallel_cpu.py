"""The exchange logic of the vocabulary-parallel step on CPU: two gloo ranks,
each holding one shard of the vocabulary, run vocab_parallel.step with
float64 stand-ins for the CUDA calls (same contracts as include/lmhead.h);
the merged statistics, the all-reduced dX and the per-rank dW rows must equal
the whole-vocabulary oracle."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


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
            r[i] = (m, np.exp(x[i] - m).sum(), x[i, y - off] if own else 0.0, 1.0 if own else 0.0)
        rec.copy_(torch.from_numpy(r).float())

    @staticmethod
    def ce_merge_shards(recs, target, stats, vtot, ignore, status=None):
        R = recs.double().numpy()
        out = np.zeros((R.shape[1], 4))
        for i, y in enumerate(target.tolist()):
            if y == ignore or y < 0 or y >= vtot:
                continue
            m = R[:, i, 0].max()
            d = (R[:, i, 1] * np.exp(R[:, i, 0] - m)).sum()
            xy = R[R[:, i, 3] != 0, i, 2].sum()
            out[i] = (m, d, xy, m + np.log(d) - xy)
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
                out[i, y - off] -= 1.0
            out[i] *= float(g.reshape(-1)[0])
        dl.copy_(torch.from_numpy(out).to(dl.dtype))

    @staticmethod
    def lmhead_bwd_dx(dl, W, dX, status=None):
        dX.copy_((dl.double() @ W.double()).float())

    @staticmethod
    def lmhead_bwd_dw(dl, X, dW, status=None):
        dW.copy_((dl.double().T @ X.double()).float())


def _inputs():
    g = torch.Generator().manual_seed(5)
    M, K, V = 12, 16, 40
    X = (torch.randn(M, K, generator=g)).to(torch.bfloat16)
    W = (torch.randn(V, K, generator=g) * 0.3).to(torch.bfloat16)
    t = torch.randint(0, V, (M,), generator=g)
    t[2] = -100
    return X, W, t, V


def _rank(rank, world, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from lm_head_fp32_b200 import vocab_parallel
    dist.init_process_group("gloo", rank=rank, world_size=world)
    X, W, t, V = _inputs()
    off, n = vocab_parallel.shard_bounds(V, world, rank)
    g = torch.tensor([0.5])
    stats, dX, dW, _, _ = vocab_parallel.step(X, W[off:off + n].contiguous(), t, off, V, g,
                                              ops=FakeOps)
    q.put((rank, off, stats.numpy(), dX.numpy(), dW.numpy()))
    dist.destroy_process_group()


def test_two_ranks_match_whole_vocabulary():
    import oracle
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
    assert all(p.exitcode == 0 for p in procs)
    res.sort(key=lambda r: r[0])
    X, W, t, V = _inputs()
    L = oracle.logits(X.view(torch.int16).numpy().view(np.uint16),
                      W.view(torch.int16).numpy().view(np.uint16))
    Lf = oracle.round_f32(L)
    ref, code = oracle.ce_fwd(Lf, t.numpy())
    dl = oracle.round_bf16(oracle.ce_bwd(Lf, t.numpy(), 0.5))
    ref_dx = oracle.dx(dl, W.view(torch.int16).numpy().view(np.uint16))
    ref_dw = oracle.dw(dl, X.view(torch.int16).numpy().view(np.uint16))
    for rank, off, stats, dX, dW in res:
        np.testing.assert_allclose(stats[:, 3], ref[:, 3], rtol=1e-5, atol=1e-5)
        np.testing.assert_allclose(dX, ref_dx, rtol=1e-4, atol=1e-5)
        np.testing.assert_allclose(dW, ref_dw[off:off + dW.shape[0]], rtol=1e-4, atol=1e-5)
    assert sum(r[4].shape[0] for r in res) == V


def test_shard_bounds_cover_the_vocabulary():
    from lm_head_fp32_b200 import vocab_parallel
    for V in (40, 128256, 151936, 7):
        for world in (1, 2, 3, 8):
            spans = [vocab_parallel.shard_bounds(V, world, r) for r in range(world)]
            assert spans[0][0] == 0 and sum(n for _, n in spans) == V
            for (o1, n1), (o2, _) in zip(spans, spans[1:]):
                assert o1 + n1 == o2
