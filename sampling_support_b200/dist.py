"""Row-sharded (data-parallel) use of the library across ranks.

Rows are independent, so a batch splits across ranks with no exchange on the
data path.  The only cross-rank steps are scalar reductions:

* the weighted distance loss (DeepSpec PR #87, "Purpose": the distributed
  normalisation of the weighted L1 loss is kept): the loss of the whole batch
  is sum_ranks sum_i w_i L1_i / sum_ranks sum_i w_i, and each rank's gradient
  needs the global denominator;
* the support-entropy statistic (SkyRL PR #2004, "Implementation": the
  entropy statistic joins the reduction that the replay logprob already
  uses): sum over valid rows of H_S and the count of valid rows.

The vocabulary-parallel fused head (tensor parallelism over the LM head's
vocabulary) has one real exchange: every rank's fixed-size partial record
block (per row: the shard's online statistics, its top-k candidates and the
target logit) is all-gathered, and every rank merges the blocks.

The library performs no collective itself; these helpers call it and reduce
the scalars with torch.distributed (NCCL on GPUs).  Every rank must call them
in the same order.
"""

from __future__ import annotations

import torch
import torch.distributed as dist

from . import _binding as B


class LibraryOps:
    """The per-rank steps, run by libvs.so."""

    @staticmethod
    def lmhead_partial(hidden, weight_shard, vocab_begin, vocab_total, targets, temperature,
                       top_k):
        return B.fused_lmhead_partial(hidden, weight_shard, vocab_begin, vocab_total, targets,
                                      temperature, top_k)

    @staticmethod
    def lmhead_merge(partials, rows, vocab_total, targets, temperature, top_k, top_p, min_p):
        return B.fused_lmhead_merge(partials, rows, vocab_total, targets, temperature, top_k,
                                    top_p, min_p)

    @staticmethod
    def weight_sum(rows, row_weight, device):
        return B.l1_weight_sum(rows, row_weight, device=device)

    @staticmethod
    def l1_distance(draft, target, row_weight, global_weight_sum, want_grad, grad_dtype):
        return B.l1_distance(draft, target, row_weight, want_loss=True, want_grad=want_grad,
                             grad_dtype=grad_dtype, global_weight_sum=global_weight_sum)


def sharded_l1_distance(draft, target, row_weight=None, group=None, want_grad=True,
                        grad_dtype=torch.float32, ops=LibraryOps):
    """Distance, accept rate, loss and draft gradient of this rank's rows of a
    row-sharded batch.

    Steps: this rank's weight sum (fp64) -> all-reduce -> the distance call
    with the global sum (gradient normalised by it) -> all-reduce of
    (numerator, denominator, loss contribution).  Returns the library's
    per-row outputs plus "loss_global" (the batch loss), "num_global" and
    "den_global" (float64 tensors of one element)."""
    rows = draft.shape[0]
    wsum = ops.weight_sum(rows, row_weight, draft.device)
    dist.all_reduce(wsum, group=group)
    out = ops.l1_distance(draft, target, row_weight, wsum, want_grad, grad_dtype)
    parts = out["loss"][:3].to(torch.float64)
    dist.all_reduce(parts, group=group)
    out["num_global"], out["den_global"], out["loss_global"] = parts[0:1], parts[1:2], parts[2:3]
    out["weight_sum_global"] = wsum
    return out


def sharded_entropy_mean(entropy_sum, valid_count, group=None):
    """Mean support entropy over the valid rows of all ranks from each rank's
    vs_score_fwd reduction outputs (entropy_sum float64 [1], valid_count
    int32 [1]); 0 when no rank has a valid row."""
    t = torch.cat([entropy_sum.to(torch.float64).reshape(1),
                   valid_count.to(torch.float64).reshape(1)])
    dist.all_reduce(t, group=group)
    return torch.where(t[1] > 0, t[0] / t[1].clamp(min=1.0), torch.zeros_like(t[0]))


def tp_fused_lmhead_score(hidden, weight_shard, vocab_begin, vocab_total, targets, temperature,
                          top_k, top_p, min_p, group=None, ops=LibraryOps):
    """Fused-head scoring with the vocabulary split across the ranks of
    `group`: rank r holds weight rows [vocab_begin, vocab_begin + rows of
    weight_shard), and the shards are in rank order.  Every rank returns the
    outputs of fused_lmhead_score over the whole vocabulary.

    Steps: this rank's partial block -> all-gather of the blocks (rank
    order) -> the merge."""
    block = ops.lmhead_partial(hidden, weight_shard, vocab_begin, vocab_total, targets,
                               temperature, top_k)
    world = dist.get_world_size(group)
    parts = [torch.empty_like(block) for _ in range(world)]
    dist.all_gather(parts, block, group=group)
    gathered = torch.stack(parts)
    return ops.lmhead_merge(gathered, hidden.shape[0], vocab_total, targets, temperature, top_k,
                            top_p, min_p)
