"""Failure detection and stream behaviour on the GPU.

* A bounded pipeline wait is made to run out on purpose (a barrier nothing
  arrives at): the kernel unwinds, reports LMH_DEV_PIPE_TIMEOUT through the
  status word, and the context stays usable.  No fault, trap or hang.
* The whole five-call step is captured in a CUDA graph and replayed: the calls
  only enqueue stream work (no allocation, no synchronisation), and replays
  reproduce the eager results bit for bit.
"""
import pytest
import torch

from lm_head_fp32_b200 import lmhead, synth

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
    out = torch.empty((16, 256), dtype=torch.float32, device=DEV)
    st2 = torch.zeros(1, dtype=torch.int32, device=DEV)
    lmhead.lmhead_fwd(X.to(DEV), W.to(DEV), out, st2)
    torch.cuda.synchronize()
    assert int(st2.item()) == 0
    ref = (X.to(torch.int64) @ W.to(torch.int64).T).to(torch.float32)
    assert torch.equal(out.cpu(), ref)


def test_whole_step_in_a_cuda_graph():
    cfg = synth.GemmConfig("graph_step", 512, 1024, 8192, "normal", ignore_frac=0.02)
    X, W, t = cfg.make()
    M, K, V = cfg.M, cfg.K, cfg.V
    Xd, Wd, td = X.to(DEV), W.to(DEV), t.to(DEV)
    g = torch.tensor([cfg.grad_scalar(t)], dtype=torch.float32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    bufs = dict(logits=torch.empty((M, V), device=DEV), stats=torch.empty((M, 4), device=DEV),
                dl=torch.empty((M, V), dtype=torch.bfloat16, device=DEV),
                dX=torch.empty((M, K), device=DEV), dW=torch.empty((V, K), device=DEV))

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
