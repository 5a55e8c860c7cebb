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

from typing import Optional

import torch
import torch.distributed as dist

from . import lmhead as _lmhead


def shard_bounds(vocab_total: int, world: int, rank: int, multiple: int = 8):
    """[offset, offset + size) of rank's shard: near-equal sizes, each a
    multiple of `multiple` entries except possibly the last."""
    per = -(-vocab_total // world)
    per = -(-per // multiple) * multiple
    off = min(rank * per, vocab_total)
    return off, min(per, vocab_total - off)


def step(X: torch.Tensor, W_shard: torch.Tensor, target: torch.Tensor, vocab_offset: int,
         vocab_total: int, grad_loss: torch.Tensor, group=None, ignore_index: int = -100,
         status: Optional[torch.Tensor] = None, ops=None):
    """One vocabulary-parallel forward + backward on this rank.

    Returns (stats[M,4] of the whole vocabulary, dX[M,K] summed over ranks,
    dW_shard[V_r,K], logits_shard, dl_shard)."""
    ops = ops or _lmhead
    M, K = X.shape
    Vr = W_shard.shape[0]
    dev = X.device
    world = dist.get_world_size(group) if dist.is_initialized() else 1

    logits = torch.empty((M, Vr), dtype=torch.float32, device=dev)
    ops.lmhead_fwd(X, W_shard, logits, status)
    rec = torch.empty((M, 4), dtype=torch.float32, device=dev)
    ops.ce_fwd_shard(logits, target, rec, vocab_offset, vocab_total, ignore_index, status)
    if world > 1:
        parts = [torch.empty_like(rec) for _ in range(world)]
        dist.all_gather(parts, rec, group=group)
        recs = torch.stack(parts)
    else:
        recs = rec.unsqueeze(0)
    stats = torch.empty((M, 4), dtype=torch.float32, device=dev)
    ops.ce_merge_shards(recs.contiguous(), target, stats, vocab_total, ignore_index, status)

    dl = torch.empty((M, Vr), dtype=torch.bfloat16, device=dev)
    ops.ce_bwd_shard(logits, target, stats, grad_loss, dl, vocab_offset, vocab_total,
                     ignore_index, status)
    dX = torch.empty((M, K), dtype=torch.float32, device=dev)
    ops.lmhead_bwd_dx(dl, W_shard, dX, status)
    if world > 1:
        dist.all_reduce(dX, op=dist.ReduceOp.SUM, group=group)
    dW = torch.empty((Vr, K), dtype=torch.float32, device=dev)
    ops.lmhead_bwd_dw(dl, X, dW, status)
    return stats, dX, dW, logits, dl
