"""Failure detection and stream behaviour on the GPU.

* A bounded pipeline wait is made to run out on purpose (a barrier nothing
  arrives at): the kernel unwinds, reports LMH_DEV_PIPE_TIMEOUT through the
  status word, and the context stays usable.  No fault, trap or hang.
* The same for the vocabulary GEMM itself: with every pipeline wait limited
  to 1 ns its waits run out, each CTA lets its issued operand copies land,
  drains its MMAs, frees tensor memory and sets the status bit; the next
  normal call on the same buffers is bit-exact.
* The whole five-call step is captured in a CUDA graph and replayed: the calls
  only enqueue stream work (no allocation, no synchronisation), and replays
  reproduce the eager results bit for bit.
* Two independent steps run at the same time on two streams (the library
  holds no state between calls apart from cached driver handles) and give
  the bits each gives alone; the dX split of the last wave is among them.
"""
import pytest
import torch

from lm_head_fp32_b200 import lmhead, synth
from helpers import guarded_empty, guarded_full

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_watchdog_wait_runs_out_and_context_survives():
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    lmhead.watchdog_selftest(status, limit_us=2000)
    torch.cuda.synchronize()
    assert int(status.item()) & lmhead.DEV_PIPE_TIMEOUT
    # the context is still usable: a normal call afterwards succeeds
    X = synth.int_bf16((16, 64), 1)
    W = synth.int_bf16((256, 64), 2)
    out = guarded_empty((16, 256), torch.float32)
    st2 = torch.zeros(1, dtype=torch.int32, device=DEV)
    lmhead.lmhead_fwd(X.to(DEV), W.to(DEV), out, st2)
    torch.cuda.synchronize()
    assert int(st2.item()) == 0
    ref = (X.to(torch.int64) @ W.to(torch.int64).T).to(torch.float32)
    assert torch.equal(out.cpu(), ref)


def test_gemm_wait_runs_out_unwinds_and_next_call_is_exact():
    # 64 tokens: single-CTA tiles (two CTAs resident per SM, one tile each);
    # a tile's mainloop over K = 8192 takes tens of microseconds, far beyond a
    # 1 ns limit, so the epilogue's first wait for its accumulator runs out
    M, K, V = 64, 8192, 32768
    X = synth.int_bf16((M, K), 11)
    W = synth.int_bf16((V, K), 12)
    Xd, Wd = X.to(DEV), W.to(DEV)
    out = guarded_full((M, V), float("nan"))
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    lmhead.gemm_watchdog_selftest(Xd, Wd, out, status, limit_ns=1)
    torch.cuda.synchronize()
    assert int(status.item()) & lmhead.DEV_PIPE_TIMEOUT
    st2 = torch.zeros(1, dtype=torch.int32, device=DEV)
    lmhead.lmhead_fwd(Xd, Wd, out, st2)
    torch.cuda.synchronize()
    assert int(st2.item()) == 0
    # integers in [-8, 8] with K * 64 < 2^24: every partial sum is exact
    ref = (X.double() @ W.double().T).to(torch.float32)
    assert torch.equal(out.cpu(), ref)


def test_whole_step_in_a_cuda_graph():
    cfg = synth.GemmConfig("graph_step", 512, 1024, 8192, "normal", ignore_frac=0.02)
    X, W, t = cfg.make()
    M, K, V = cfg.M, cfg.K, cfg.V
    Xd, Wd, td = X.to(DEV), W.to(DEV), t.to(DEV)
    g = torch.tensor([cfg.grad_scalar(t)], dtype=torch.float32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    bufs = dict(logits=guarded_empty((M, V)), stats=guarded_empty((M, 4)),
                dl=guarded_empty((M, V), torch.bfloat16),
                dX=guarded_empty((M, K)), dW=guarded_empty((V, K)))

    def step():
        lmhead.lmhead_fwd(Xd, Wd, bufs["logits"], status)
        lmhead.ce_fwd(bufs["logits"], td, bufs["stats"], -100, status)
        lmhead.ce_bwd(bufs["logits"], td, bufs["stats"], g, bufs["dl"], -100, status)
        lmhead.lmhead_bwd_dx(bufs["dl"], Wd, bufs["dX"], status)
        lmhead.lmhead_bwd_dw(bufs["dl"], Xd, bufs["dW"], status)

    step()                                   # eager
    torch.cuda.synchronize()
    eager = {k: v.clone() for k, v in bufs.items()}
    for v in bufs.values():
        v.zero_()
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph):
            step()
    torch.cuda.current_stream().wait_stream(side)
    for _ in range(2):
        for v in bufs.values():
            v.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        for k in bufs:
            assert torch.equal(bufs[k], eager[k]), k
    del graph


def _step_buffers(M, K, V, seed):
    cfg = synth.GemmConfig(f"concurrent_{seed}", M, K, V, "normal", ignore_frac=0.02, seed=seed)
    X, W, t = cfg.make()
    g = torch.tensor([cfg.grad_scalar(t)], dtype=torch.float32, device=DEV)
    ins = dict(X=X.to(DEV), W=W.to(DEV), t=t.to(DEV), g=g)
    outs = dict(logits=guarded_empty((M, V)), stats=guarded_empty((M, 4)),
                dl=guarded_empty((M, V), torch.bfloat16),
                dX=guarded_empty((M, K)), dW=guarded_empty((V, K)))
    return ins, outs


def _run_step(ins, outs, status, stream):
    lmhead.lmhead_fwd(ins["X"], ins["W"], outs["logits"], status, stream)
    lmhead.ce_fwd(outs["logits"], ins["t"], outs["stats"], -100, status, stream)
    lmhead.ce_bwd(outs["logits"], ins["t"], outs["stats"], ins["g"], outs["dl"], -100, status, stream)
    lmhead.lmhead_bwd_dx(outs["dl"], ins["W"], outs["dX"], status, stream)
    lmhead.lmhead_bwd_dw(outs["dl"], ins["X"], outs["dW"], status, stream)


def test_two_streams_at_once_match_each_alone():
    # 2560 tokens x K = 2048: dX's last wave is split (80 pair tiles on 74 pairs)
    cases = [(2560, 2048, 1032, 5), (300, 1024, 8200, 6)]
    bufs = [_step_buffers(*c) for c in cases]
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    alone = []
    for ins, outs in bufs:
        _run_step(ins, outs, status, None)
        torch.cuda.synchronize()
        alone.append({k: v.clone() for k, v in outs.items()})
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    for _ in range(3):
        for _, outs in bufs:
            for v in outs.values():
                v.zero_()
        torch.cuda.synchronize()
        for (ins, outs), s in zip(bufs, streams):
            _run_step(ins, outs, status, s)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        for (_, outs), ref in zip(bufs, alone):
            for k in outs:
                assert torch.equal(outs[k], ref[k]), k

