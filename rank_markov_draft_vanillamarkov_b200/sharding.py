"""Splitting the head's work across GPUs (one process per GPU).

The forward entry points are data-parallel with no exchange step:
teacher-forced rows are independent, and so are the blocks of the sampler
(each block's chain depends only on its own earlier tokens). So N GPUs hold
replicas of W1/W2 and each processes a contiguous slice of rows or blocks; no
collective is needed on the data path. These helpers compute the slices.

Training is the one place with a real exchange: every rank's rows contribute
to the same W1/W2 gradients, so the per-rank gradients are summed across the
ranks (an all-reduce; NCCL over NVLink on GPUs) before any update.
"""
from __future__ import annotations

from typing import Tuple

MASK64 = (1 << 64) - 1


def shard_range(n: int, rank: int, world: int) -> Tuple[int, int]:
    """Contiguous [start, stop) slice of n units for `rank` of `world`; sizes
    differ by at most one and the slices tile [0, n) in rank order."""
    if world <= 0 or not 0 <= rank < world:
        raise ValueError("bad rank/world")
    if n < 0:
        raise ValueError("negative size")
    return n * rank // world, n * (rank + 1) // world


def shard_seed(seed: int, first_block: int) -> int:
    """Philox seed of a shard whose first block has global index `first_block`.

    The noise counter holds the LOCAL block index, so two shards given one seed
    would draw the same noise for their block 0. Adding the shard's first
    global block index to the key's high word gives every shard its own
    stream. Greedy sampling is unaffected; temperature sampling of a sharded
    batch then draws from the same distribution as an unsharded call, but not
    the same draws."""
    return (seed + (first_block << 32)) & MASK64


def apply_block_logits_shard(head, base_logits, token_ids, rank: int, world: int):
    """This rank's slice of the leading (batch) axis, corrected."""
    lo, hi = shard_range(base_logits.shape[0], rank, world)
    return head.apply_block_logits(base_logits[lo:hi], token_ids=token_ids[lo:hi])


def sample_block_tokens_shard(head, base_logits, first_prev_token_ids, rank: int, world: int,
                              temperature=0.0, seed: int = 0):
    """This rank's slice of the blocks, sampled left to right."""
    lo, hi = shard_range(base_logits.shape[0], rank, world)
    return head.sample_block_tokens(base_logits[lo:hi], first_prev_token_ids=first_prev_token_ids[lo:hi],
                                    temperature=temperature, seed=shard_seed(seed, lo))


def apply_block_logits_backward_shard(head, grad_out, token_ids, rank: int, world: int, group=None):
    """Gradients of W1 and W2 (fp32, [V, r]) for the whole batch: this rank
    differentiates its slice of the leading (batch) axis, then the two
    gradients are summed over the ranks in place (torch.distributed
    all_reduce). With world == 1 no collective runs."""
    import torch.distributed as dist
    lo, hi = shard_range(grad_out.shape[0], rank, world)
    gw1, gw2 = head.apply_block_logits_backward(grad_out[lo:hi], token_ids=token_ids[lo:hi])
    if world > 1:
        dist.all_reduce(gw1, op=dist.ReduceOp.SUM, group=group)
        dist.all_reduce(gw2, op=dist.ReduceOp.SUM, group=group)
    return gw1, gw2
