"""Data-parallel exchange of the DPO head step.

Each rank scores its own pairs (both rows of a pair stay on one rank) with the
same weights. The loss is the mean over all pairs of all ranks, so each rank
folds 1/world_size into the per-row coefficients (dpo_loss's grad_scale), and
the step's one exchange is a sum all-reduce of dW (and of the loss, then divided
by world_size). dH stays on its rank. This mirrors the data-parallel replicas of
the pages' systems ("Run Distributed Full-Model DPO with PyTorch FSDP", Step 1;
Megatron-Bridge PR 6092, the DP replicas of its results), at the LM head.
"""
from __future__ import annotations


def grad_scale(world_size: int, accumulation_steps: int = 1) -> float:
    """grad_scale for dpo_loss so that summed per-rank gradients are those of the global mean."""
    return 1.0 / (world_size * accumulation_steps)


def allreduce_step(dW, loss, group=None):
    """Sum dW over ranks in place; turn the per-rank mean losses into the global mean."""
    import torch.distributed as dist
    ws = dist.get_world_size(group)
    dist.all_reduce(dW, group=group)
    dist.all_reduce(loss, group=group)
    loss.mul_(1.0 / ws)
