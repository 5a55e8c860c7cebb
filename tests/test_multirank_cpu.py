"""Host logic of the N > 1 bench path on CPU: two gloo ranks, each an
independent replica (no collective on the data path); the job's device time is
the maximum over ranks and the throughput counts every rank's tokens."""
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
