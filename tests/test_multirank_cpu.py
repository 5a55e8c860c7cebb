"""Host logic of the N > 1 bench paths on CPU, two gloo ranks each.

Replicas: each rank an independent replica (no collective on the data path);
the job's device time is the maximum over ranks and the throughput counts
every rank's tokens.

Vocabulary-parallel (--parallel vocab): each rank holds its shard of W and the
same batch; the step's all-gather and all-reduce run over the process group
(float64 stand-ins for the CUDA calls), every rank ends with the
whole-vocabulary statistics and the summed dX, and the line counts the batch
once (strong scaling) over the slowest rank's time."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    w, r, local, pg = bench.dist_setup(None)
    assert (w, r) == (world, rank) and pg is not None
    mine = 10.0 + 5.0 * rank                     # per-rank summed step time (ms)
    job = bench.max_over_ranks(mine, pg, "cpu")
    bench.barrier(pg)
    q.put((rank, job))
    pg.destroy_process_group()


def test_two_gloo_ranks_take_max_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    res = dict(q.get(timeout=5) for _ in range(2))
    assert res == {0: 15.0, 1: 15.0}


def test_single_rank_needs_no_process_group(monkeypatch):
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    sys.path.insert(0, ROOT)
    import bench
    w, r, local, pg = bench.dist_setup(None)
    assert (w, r, pg) == (1, 0, None)
    assert bench.max_over_ranks(3.5, pg, "cpu") == 3.5


def _vocab_rank(rank, world, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import torch
    import bench
    from helpers import FakeOps
    from lm_head_fp32_b200 import vocab_parallel
    w, r, local, pg = bench.dist_setup(None)
    cfg = bench.lmhead_config("lmhead_12x16x40")
    X, Ws, t, off, n = bench.vocab_shard_inputs(cfg, w, r)
    g = torch.tensor([cfg.grad_scalar(t)])
    seen = []
    stats, dX, dW, _, _ = vocab_parallel.step(X, Ws, t, off, cfg.V, g, ops=FakeOps,
                                              mark=seen.append)
    assert tuple(seen) == vocab_parallel.STAGES
    job = bench.max_over_ranks(100.0 + 20.0 * r, pg, "cpu")   # summed step ms
    stage_ms = {s: 1.0 for s in vocab_parallel.STAGES}
    peaks = dict(bench.FALLBACK_PEAKS)
    line = bench.vocab_line(cfg, w, 10, 3, job, stage_ms, {}, int((t != -100).sum()), peaks,
                            "fallback", n)
    q.put((r, off, n, X.float().sum().item(), stats.numpy(), dX.numpy(), line))
    pg.destroy_process_group()


def test_vocab_parallel_bench_host_logic():
    import numpy as np
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_vocab_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=180) for _ in range(2)), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    (r0, off0, n0, xs0, st0, dx0, line0), (r1, off1, n1, xs1, st1, dx1, line1) = res
    assert (off0, off0 + n0) == (0, off1) and off1 + n1 == 40    # the shards tile V
    assert xs0 == xs1                                            # one batch for all ranks
    assert np.array_equal(st0, st1) and np.array_equal(dx0, dx1)  # exchanged results agree
    # the whole-vocabulary loss, from a float64 restatement on one rank
    import bench
    cfg = bench.lmhead_config("lmhead_12x16x40")
    X, W, t = cfg.make()
    L = (X.double() @ W.double().T).float().double().numpy()
    for i, y in enumerate(t.tolist()):
        if y == -100:
            assert st0[i, 3] == 0
            continue
        m = L[i].max()
        ref = m + np.log(np.exp(L[i] - m).sum()) - L[i, y]
        assert abs(st0[i, 3] - ref) <= 1e-5 * abs(ref) + 1e-5
    # strong scaling: 12 tokens per step over the slowest rank's 120 ms for 10 steps
    assert line0["scaling"] == "strong" and line0["n_gpus"] == 2
    assert abs(line0["value"] - 12 * 10 / 0.120) < 1e-6
    assert line0["config"]["parallelism"] == "vocab2" and line0["config"]["nccl_ranks"] == 2
    assert line0["config"]["vocab_rows_per_rank"] == n0
