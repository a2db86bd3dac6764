"""Multi-GPU plumbing of the layer: token-sharded data parallelism.

Every rank holds the full layer (weights replicated) and routes its own share
of the step's tokens; everything on the path is per token except the load
over the whole batch of the step, which the bias update needs (kbwen.com
DeepSeek tag page, "A bias term for each expert": the load is monitored over
the whole batch of the step).  That is the one exchange: the per-expert
counts are summed over the ranks (an all-reduce of E int32 over NCCL) and
every rank then applies the identical update with the global token count, so
the biases stay bit-identical without ever being sent.
"""
from __future__ import annotations

import torch


def shard_step(step: int, rank: int, world: int) -> int:
    """Token-draw index of this rank's shard of step ``step`` (feeds
    ``inputs.make_tokens``); shards of one step never repeat a draw."""
    return step * world + rank


def global_token_count(tokens_per_rank: int, world: int) -> int:
    return tokens_per_rank * world


def allreduce_counts(counts: torch.Tensor, group=None) -> torch.Tensor:
    """Sum the per-expert counts of all ranks in place (no-op on one rank)."""
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(counts, op=dist.ReduceOp.SUM, group=group)
    return counts
