"""The autograd entry (lm_head_fp32_b200.loss.lm_head_cross_entropy) against
the C-ABI calls it marshals: the same kernels on the same inputs, so the
per-token loss and the gradients must match bit for bit; plus one end-to-end
check of the loss against the FP64 oracle on integer operands (exact FP32
logits)."""
import numpy as np
import pytest
import torch

import oracle
from lm_head_fp32_b200 import lmhead, synth
from lm_head_fp32_b200.loss import lm_head_cross_entropy
from helpers import assert_abs_close, bits, loss_tol

pytestmark = pytest.mark.gpu
DEV = "cuda"


def inputs(M, K, V, seed, ignore_frac=0.1):
    X = synth.normal_bf16((M, K), 1.0, seed).to(DEV)
    W = synth.normal_bf16((V, K), 0.02, seed + 1).to(DEV)
    t = synth.targets(M, V, ignore_frac, seed + 2).to(DEV)
    return X, W, t


def direct(X, W, t, g):
    """The five calls with grad_loss g (one element or one per token)."""
    M, V = X.shape[0], W.shape[0]
    logits = torch.empty((M, V), dtype=torch.float32, device=DEV)
    stats = torch.empty((M, 4), dtype=torch.float32, device=DEV)
    lmhead.lmhead_fwd(X, W, logits)
    lmhead.ce_fwd(logits, t, stats)
    dl = torch.empty((M, V), dtype=torch.bfloat16, device=DEV)
    lmhead.ce_bwd(logits, t, stats, g.to(DEV, torch.float32).contiguous(), dl)
    dX = lmhead.lmhead_bwd_dx(dl, W, torch.empty_like(X))
    dW = lmhead.lmhead_bwd_dw(dl, X, torch.empty_like(W))
    return stats[:, 3], dl, dX, dW


@pytest.mark.parametrize("fused", [True, False])
@pytest.mark.parametrize("M,K,V", [(300, 264, 1000), (17, 72, 32776), (512, 1024, 8200)])
def test_loss_and_grads_match_the_calls(fused, M, K, V):
    X, W, t = inputs(M, K, V, 7 + M)
    Xr, Wr = X.clone().requires_grad_(), W.clone().requires_grad_()
    loss = lm_head_cross_entropy(Xr, Wr, t, fused=fused)
    loss.sum().backward()            # every token's gradient is 1: the one-element path
    ref_loss, _, ref_dX, ref_dW = direct(X, W, t, torch.ones(1))
    assert loss.dtype == torch.float32 and loss.shape == (M,)
    if fused:
        # the fused statistics merge in another order: within the loss tolerance
        assert_abs_close(loss.detach().double().cpu().numpy(), ref_loss.double().cpu().numpy(),
                         2 * loss_tol(ref_loss.double().cpu().numpy()), "fused loss")
    else:
        assert torch.equal(loss.detach(), ref_loss)
    if not fused:
        assert torch.equal(Xr.grad, ref_dX) and torch.equal(Wr.grad, ref_dW)
    assert Xr.grad.dtype == torch.bfloat16 and Wr.grad.dtype == torch.bfloat16


def test_mean_and_weighted_losses():
    """loss.mean(): one gradient 1/M for every token; a weighted sum: one
    gradient per token.  Both equal ce_bwd called with the same gradients."""
    M, K, V = 200, 520, 4104
    X, W, t = inputs(M, K, V, 31)
    Xr, Wr = X.clone().requires_grad_(), W.clone().requires_grad_()
    lm_head_cross_entropy(Xr, Wr, t, fused=False).mean().backward()
    _, _, dX, dW = direct(X, W, t, torch.full((1,), 1.0 / M))
    assert torch.equal(Xr.grad, dX) and torch.equal(Wr.grad, dW)
    w = torch.rand(M, generator=torch.Generator().manual_seed(5)).to(DEV)
    Xr.grad = Wr.grad = None
    (lm_head_cross_entropy(Xr, Wr, t, fused=False) * w).sum().backward()
    _, _, dX, dW = direct(X, W, t, w)
    assert torch.equal(Xr.grad, dX) and torch.equal(Wr.grad, dW)


def test_main_grad_accumulates_in_fp32():
    M, K, V = 300, 264, 1000
    X, W, t = inputs(M, K, V, 41)
    main = (torch.randn((V, K), generator=torch.Generator().manual_seed(6)) * 1e-3).to(DEV)
    expect = main.clone()
    Xr, Wr = X.clone().requires_grad_(), W.clone().requires_grad_()
    lm_head_cross_entropy(Xr, Wr, t, fused=False, main_grad=main).sum().backward()
    _, dl, dX, _ = direct(X, W, t, torch.ones(1))
    lmhead.lmhead_bwd_dw_acc(dl, X, expect)
    assert Wr.grad is None
    assert torch.equal(main, expect) and torch.equal(Xr.grad, dX)


def test_loss_against_the_oracle_on_integer_operands():
    """Integer BF16 operands in [-8, 8]: the FP32 logits are exact, so the
    per-token loss is within the loss tolerance of the FP64 oracle's."""
    M, K, V = 64, 128, 2056
    X = synth.int_bf16((M, K), 51)
    W = synth.int_bf16((V, K), 52)
    t = synth.targets(M, V, 0.1, 53)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    loss = lm_head_cross_entropy(X.to(DEV), W.to(DEV), t.to(DEV), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    exact = oracle.round_f32(oracle.logits(bits(X), bits(W)))
    ref, _ = oracle.ce_fwd(exact, t.numpy(), -100)
    assert_abs_close(loss.double().cpu().numpy(), ref[:, 3], loss_tol(ref[:, 3]), "loss")


def test_bad_target_sets_the_status_bit():
    M, K, V = 8, 64, 512
    X, W, t = inputs(M, K, V, 61, 0.0)
    t[3] = V + 5
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    loss = lm_head_cross_entropy(X, W, t, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & lmhead.DEV_BAD_TARGET
    assert float(loss[3]) == 0.0
