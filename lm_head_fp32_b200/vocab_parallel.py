"""Vocabulary-parallel LM-head loss step across devices.

The vocabulary weights W[V,K] are split by rows across the ranks of a process
group (rank r holds entries [offset_r, offset_r + V_r)), as Megatron's
VocabParallelCrossEntropy splits the logits (TransformerEngine #2325,
"Description").  One step on rank r:

  logits_r = X . W_r^T                      lmhead_fwd
  rec_r    = per-row (m_r, d_r, x_y?, own?) ce_fwd_shard
  recs     = all-gather of rec_r            the only exchange of the forward
  stats    = merge of recs                  ce_merge_shards (same on every rank)
  dl_r     = (softmax - onehot) * g         ce_bwd_shard
  dX       = sum_r dl_r . W_r               lmhead_bwd_dx + all-reduce (sum)
  dW_r     = dl_r^T . X                     lmhead_bwd_dw (local, no exchange)

This module only sequences the library calls and the two collectives; every
arithmetic step runs in the library's kernels.  `ops` defaults to the CUDA
binding and exists so that the sequencing can be exercised without a GPU.
"""
from __future__ import annotations

from typing import Callable, Optional

import torch
import torch.distributed as dist

from . import lmhead as _lmhead


def shard_bounds(vocab_total: int, world: int, rank: int, multiple: int = 8):
    """[offset, offset + size) of rank's shard: near-equal sizes, each a
    multiple of `multiple` entries except possibly the last.  When the
    vocabulary is small for the world size the last ranks' shards are empty
    (size 0); step() handles those."""
    per = -(-vocab_total // world)
    per = -(-per // multiple) * multiple
    off = min(rank * per, vocab_total)
    return off, min(per, vocab_total - off)


STAGES = ("lmhead_fwd", "ce_fwd_shard", "all_gather", "ce_merge_shards", "ce_bwd_shard",
          "lmhead_bwd_dx", "all_reduce", "lmhead_bwd_dw")


def step(X: torch.Tensor, W_shard: torch.Tensor, target: torch.Tensor, vocab_offset: int,
         vocab_total: int, grad_loss: torch.Tensor, group=None, ignore_index: int = -100,
         status: Optional[torch.Tensor] = None, ops=None,
         mark: Optional[Callable[[str], None]] = None):
    """One vocabulary-parallel forward + backward on this rank.

    `mark`, if given, is called with each name of STAGES, in that order, right
    after that stage has been enqueued (a timing hook).

    Returns (stats[M,4] of the whole vocabulary, dX[M,K] summed over ranks,
    dW_shard[V_r,K], logits_shard, dl_shard)."""
    ops = ops or _lmhead
    mark = mark or (lambda name: None)
    M, K = X.shape
    Vr = W_shard.shape[0]
    dev = X.device
    world = dist.get_world_size(group) if dist.is_initialized() else 1

    logits = torch.empty((M, Vr), dtype=torch.float32, device=dev)
    rec = torch.empty((M, 4), dtype=torch.float32, device=dev)
    if Vr > 0:
        ops.lmhead_fwd(X, W_shard, logits, status)
        mark("lmhead_fwd")
        ops.ce_fwd_shard(logits, target, rec, vocab_offset, vocab_total, ignore_index, status)
        mark("ce_fwd_shard")
    else:
        # an empty shard contributes the neutral record (no maximum, no mass,
        # no target) and no gradient, but still joins both collectives, so
        # that every rank takes the same steps
        rec.zero_()
        rec[:, 0] = float("-inf")
        mark("lmhead_fwd")
        mark("ce_fwd_shard")
    if world > 1:
        recs = torch.empty((world * M, 4), dtype=torch.float32, device=dev)
        dist.all_gather_into_tensor(recs, rec, group=group)
        recs = recs.view(world, M, 4)
    else:
        recs = rec.unsqueeze(0)
    mark("all_gather")
    stats = torch.empty((M, 4), dtype=torch.float32, device=dev)
    ops.ce_merge_shards(recs, target, stats, vocab_total, ignore_index, status)
    mark("ce_merge_shards")

    dl = torch.empty((M, Vr), dtype=torch.bfloat16, device=dev)
    dX = torch.empty((M, K), dtype=torch.float32, device=dev)
    if Vr > 0:
        ops.ce_bwd_shard(logits, target, stats, grad_loss, dl, vocab_offset, vocab_total,
                         ignore_index, status)
        mark("ce_bwd_shard")
        ops.lmhead_bwd_dx(dl, W_shard, dX, status)
    else:
        mark("ce_bwd_shard")
        dX.zero_()
    mark("lmhead_bwd_dx")
    if world > 1:
        dist.all_reduce(dX, op=dist.ReduceOp.SUM, group=group)
    mark("all_reduce")
    dW = torch.empty((Vr, K), dtype=torch.float32, device=dev)
    if Vr > 0:
        ops.lmhead_bwd_dw(dl, X, dW, status)
    mark("lmhead_bwd_dw")
    return stats, dX, dW, logits, dl
