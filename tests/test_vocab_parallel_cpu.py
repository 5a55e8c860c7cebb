"""The exchange logic of the vocabulary-parallel step on CPU: two or three gloo
ranks, each holding one shard of the vocabulary (possibly an empty one), run
vocab_parallel.step with
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

from helpers import FakeOps

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _inputs(V=40):
    g = torch.Generator().manual_seed(5)
    M, K = 12, 16
    X = (torch.randn(M, K, generator=g)).to(torch.bfloat16)
    W = (torch.randn(V, K, generator=g) * 0.3).to(torch.bfloat16)
    t = torch.randint(0, V, (M,), generator=g)
    t[2] = -100
    return X, W, t, V


def _rank(rank, world, port, q, V=40):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from lm_head_fp32_b200 import vocab_parallel
    dist.init_process_group("gloo", rank=rank, world_size=world)
    X, W, t, V = _inputs(V)
    off, n = vocab_parallel.shard_bounds(V, world, rank)
    g = torch.tensor([0.5])
    stats, dX, dW, _, _ = vocab_parallel.step(X, W[off:off + n].contiguous(), t, off, V, g,
                                              ops=FakeOps)
    q.put((rank, off, stats.numpy(), dX.numpy(), dW.numpy()))
    dist.destroy_process_group()


def _run_ranks(world, V):
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q, V)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
    assert all(p.exitcode == 0 for p in procs)
    res.sort(key=lambda r: r[0])
    return res


@pytest.mark.parametrize("world,V", [(2, 40), (3, 16)])
def test_ranks_match_whole_vocabulary(world, V):
    """(3, 16): shards of 8, 8 and 0 entries -- the last rank holds no
    vocabulary and must still join both collectives."""
    import oracle
    res = _run_ranks(world, V)
    X, W, t, V = _inputs(V)
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
    for V in (40, 128256, 151936, 7, 16):
        for world in (1, 2, 3, 8):
            spans = [vocab_parallel.shard_bounds(V, world, r) for r in range(world)]
            assert spans[0][0] == 0 and sum(n for _, n in spans) == V
            for (o1, n1), (o2, _) in zip(spans, spans[1:]):
                assert o1 + n1 == o2
            assert all(n >= 0 for _, n in spans)
    # small vocabularies leave trailing ranks empty (handled by step())
    assert [vocab_parallel.shard_bounds(16, 3, r)[1] for r in range(3)] == [8, 8, 0]
    assert [vocab_parallel.shard_bounds(40, 8, r)[1] for r in range(8)] == [8] * 5 + [0] * 3
