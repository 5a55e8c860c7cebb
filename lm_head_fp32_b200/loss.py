"""PyTorch autograd entry to the LM-head loss path: the per-token
cross-entropy of logits = X . W^T, kept as FP32 logits (Megatron-LM PR #6252
"Add mixed-precision (FP32) LM output logits", "What does this PR do?"), with
the cross-entropy forward saving only {m, d, x_y, loss} per token and the
backward computed in FP32 and cast to BF16 at the end (TransformerEngine
#2325 "[Pytorch] change fused cross entropy backward grad to fp32 and reduce
one read", "Description").

Argument marshalling only, like the binding it calls: the forward runs
lmhead_fwd_ce (or lmhead_fwd + ce_fwd), the backward ce_bwd, lmhead_bwd_dx and
lmhead_bwd_dw (or lmhead_bwd_dw_acc into a caller's FP32 main gradient).
The loss is per token, 0 on ignored tokens; averaging over the tokens that
count is the caller's, e.g. ``loss.sum() / (target != ignore_index).sum()``.
Device conditions (a target outside [0, V) that is not ignore_index) are OR-ed
into ``status`` when one is given, as in the C ABI; nothing synchronises.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import lmhead


def _check_inputs(X: torch.Tensor, W: torch.Tensor, target: torch.Tensor):
    if not (X.is_cuda and W.is_cuda and target.is_cuda):
        raise ValueError("X, W and target must be CUDA tensors (the library has no CPU path)")
    if X.dtype != torch.bfloat16 or W.dtype != torch.bfloat16:
        raise TypeError("X and W must be bfloat16")
    if target.dtype != torch.int64:
        raise TypeError("target must be int64")
    if X.dim() != 2 or W.dim() != 2 or target.dim() != 1 or X.shape[1] != W.shape[1] \
            or target.shape[0] != X.shape[0]:
        raise ValueError("expected X [M,K], W [V,K], target [M]")


class _LMHeadCrossEntropy(torch.autograd.Function):
    @staticmethod
    def forward(ctx, X, W, target, ignore_index, fused, main_grad, status):
        M, V = X.shape[0], W.shape[0]
        dev = X.device
        if status is None:
            status = torch.zeros(1, dtype=torch.int32, device=dev)
        logits = torch.empty((M, V), dtype=torch.float32, device=dev)
        stats = torch.empty((M, 4), dtype=torch.float32, device=dev)
        if fused:
            ws = torch.empty(max(lmhead.lmhead_fwd_ce_workspace_bytes(M, V), 16),
                             dtype=torch.uint8, device=dev)
            lmhead.lmhead_fwd_ce(X, W, target, logits, stats, ws, ignore_index, status)
        else:
            lmhead.lmhead_fwd(X, W, logits, status)
            lmhead.ce_fwd(logits, target, stats, ignore_index, status)
        ctx.save_for_backward(X, W, target, logits, stats, status)
        ctx.ignore_index = ignore_index
        ctx.main_grad = main_grad
        return stats[:, 3].clone()

    @staticmethod
    def backward(ctx, grad_loss):
        X, W, target, logits, stats, status = ctx.saved_tensors
        M, V = logits.shape
        # one element when every token has the same gradient (loss.sum(),
        # loss.mean()), which ce_bwd broadcasts; otherwise one per token
        if grad_loss.dim() == 1 and grad_loss.shape[0] > 1 and grad_loss.stride(0) == 0:
            g = grad_loss[:1]
        else:
            g = grad_loss
        g = g.to(torch.float32).contiguous()
        dl = torch.empty((M, V), dtype=torch.bfloat16, device=X.device)
        lmhead.ce_bwd(logits, target, stats, g, dl, ctx.ignore_index, status)
        dX = dW = None
        if ctx.needs_input_grad[0]:
            dX = lmhead.lmhead_bwd_dx(dl, W, torch.empty_like(X), status)
        if ctx.main_grad is not None:
            lmhead.lmhead_bwd_dw_acc(dl, X, ctx.main_grad, status)
        elif ctx.needs_input_grad[1]:
            dW = lmhead.lmhead_bwd_dw(dl, X, torch.empty_like(W), status)
        return dX, dW, None, None, None, None, None


def lm_head_cross_entropy(X: torch.Tensor, W: torch.Tensor, target: torch.Tensor,
                          ignore_index: int = lmhead.IGNORE_INDEX, fused: bool = True,
                          main_grad: Optional[torch.Tensor] = None,
                          status: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Per-token loss [M] (FP32) of the LM head: -log softmax(X . W^T)[target].

    X: [M, K] bfloat16 activations; W: [V, K] bfloat16 vocabulary weights;
    target: [M] int64.  ``fused`` computes the logits and the forward
    statistics in one kernel (lmhead_fwd_ce); otherwise lmhead_fwd then
    ce_fwd.  The backward gives X and W bfloat16 gradients; with
    ``main_grad`` (an FP32 [V, K] tensor) dW is added into it instead
    (lmhead_bwd_dw_acc) and W receives no gradient.  ``status``: an optional
    int32 device word that collects the device-side condition bits."""
    _check_inputs(X, W, target)
    if main_grad is not None and (main_grad.dtype != torch.float32 or
                                  tuple(main_grad.shape) != tuple(W.shape)):
        raise ValueError("main_grad must be an FP32 tensor shaped like W")
    return _LMHeadCrossEntropy.apply(X.contiguous(), W.contiguous(), target.contiguous(),
                                     int(ignore_index), bool(fused), main_grad, status)
