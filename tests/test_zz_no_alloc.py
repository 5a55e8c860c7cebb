"""lmhead_fwd_ce_noalloc: the fused logits + cross-entropy statistics call for
callers that cannot allocate device memory (its scratch is a fixed array
inside the library).

Through the C ABI, two calls in a row (different inputs, so the second call
runs over the first call's leftovers in the shared array) are checked against
lmhead_fwd_ce with a caller-provided workspace.  Both calls run the same
kernels and merge the partial statistics in the same fixed order, so the
logits and the statistics must agree bit for bit: a stale entry of the shared
array read by the second call would change the statistics.  The file is named
so that pytest collects it last; it also passes on its own in a fresh process.
"""
import pytest
import torch

from lm_head_fp32_b200 import lmhead, synth
from helpers import guarded_empty

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _inputs(seed, M, K, V):
    X = synth.normal_bf16((M, K), 1.0, seed).to(DEV)
    W = synth.normal_bf16((V, K), 0.05, seed + 1).to(DEV)
    t = synth.targets(M, V, 0.02, seed).to(DEV)
    return X, W, t


def _with_workspace(X, W, t):
    M, V = X.shape[0], W.shape[0]
    logits = guarded_empty((M, V), torch.float32)
    stats = guarded_empty((M, 4), torch.float32)
    ws = guarded_empty((lmhead.lmhead_fwd_ce_workspace_bytes(M, V),), torch.uint8)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    lmhead.lmhead_fwd_ce(X, W, t, logits, stats, ws, -100, st)
    return logits, stats, st


def _without_allocation(X, W, t):
    M, V = X.shape[0], W.shape[0]
    logits = guarded_empty((M, V), torch.float32)
    stats = guarded_empty((M, 4), torch.float32)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    lmhead.lmhead_fwd_ce_noalloc(X, W, t, logits, stats, -100, st)
    return logits, stats, st


def test_no_alloc_matches_workspace_entry_point_twice():
    # the largest problem the fixed array holds at this vocabulary: M * 2 * ceil(V/256) = 2^20
    M, K, V = 4096, 256, 32768
    for seed in (301, 302):
        X, W, t = _inputs(seed, M, K, V)
        l_ref, s_ref, st_ref = _with_workspace(X, W, t)
        l_got, s_got, st_got = _without_allocation(X, W, t)
        torch.cuda.synchronize()
        assert int(st_ref.item()) == 0 and int(st_got.item()) == 0
        assert torch.equal(l_got, l_ref)
        assert torch.equal(s_got, s_ref)


def test_no_alloc_rejects_problems_beyond_its_array():
    M, K, V = 4097, 64, 32768          # one token more than the array holds
    X, W, t = _inputs(303, M, K, V)
    logits = guarded_empty((M, V), torch.float32)
    stats = guarded_empty((M, 4), torch.float32)
    with pytest.raises(lmhead.LmhError) as e:
        lmhead.lmhead_fwd_ce_noalloc(X, W, t, logits, stats)
    assert e.value.code == lmhead.LMH_ERR_INVALID_ARG
