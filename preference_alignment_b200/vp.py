"""Vocabulary-parallel DPO head: W split by vocabulary rows across ranks.

Every rank holds the same batch (H, tokens, offsets) and a contiguous block of W's
rows; the full [V, d] head never sits on one GPU. Per step, on every rank:

1. its shard's per-position log-sum-exp and target logit (-inf when another
   shard holds the target): dpo_shard_logprob_parts;
2. an all-gather of those two [Nc] vectors (2 * Nc floats per rank, the only
   forward exchange);
3. the merge in shard order, identical on every rank: dpo_shard_combine gives the
   sequence sums, token log-probs and the backward's lse_state;
4. (policy) dpo_shard_backward with the merged lse_state: this rank's rows of dW
   (no exchange) and a partial dH; a sum all-reduce of the partial dH ([R, L, d]
   fp32) gives dH on every rank.

The pages scale the step out by sharding the model across GPUs ("Run Distributed
Full-Model DPO with PyTorch FSDP", Step 1; Megatron-Bridge PR 6092 runs tensor
parallelism); this is that split applied to the LM head, with the exchanges above
in place of gathering W. The collectives are torch.distributed calls on the current
stream; the library itself makes none.
"""
from __future__ import annotations

from preference_alignment_b200 import libdpo


def shard_range(total: int, world: int, rank: int, align: int = 256):
    """(offset, rows) of rank's contiguous shard of a `total`-row vocabulary.

    Shards are whole multiples of `align` rows (the GEMM's 256-column vocabulary
    tiles), the last one shorter, when that leaves every rank at least one row;
    otherwise the rows are split as evenly as possible. Shards are in rank order,
    disjoint, and cover [0, total).
    """
    if world < 1 or not 0 <= rank < world or total < world:
        raise ValueError("need 0 <= rank < world <= total")
    per = -(-total // world)
    per = -(-per // align) * align
    if per * (world - 1) < total:
        offset = rank * per
        return offset, min(per, total - offset)
    offset = rank * total // world
    return offset, (rank + 1) * total // world - offset


class VocabParallelHead:
    """One rank's view of a vocabulary-parallel head (shard `rank` of `world`)."""

    def __init__(self, offset: int, total: int, group=None, ops=None):
        import torch.distributed as dist
        self.offset, self.total, self.group = int(offset), int(total), group
        self.world = dist.get_world_size(group)
        self.ops = ops if ops is not None else libdpo

    def seq_logprobs(self, batch, seq_logp, tok_logp, lse_state, ws, ws_bytes=None, stream=None):
        """Full-vocabulary sums (and token log-probs / lse_state) from this rank's shard."""
        import torch
        import torch.distributed as dist
        nc = batch.n_scored
        dev = seq_logp.device
        parts = torch.empty(2, max(nc, 1), device=dev, dtype=seq_logp.dtype)
        self.ops.shard_logprob_parts(batch, self.offset, self.total, parts[0], parts[1], ws,
                                     ws_bytes=ws_bytes, stream=stream)
        # concatenated along dim 0 (the form every backend accepts), then viewed per rank
        flat = torch.empty(self.world * 2, max(nc, 1), device=dev, dtype=seq_logp.dtype)
        dist.all_gather_into_tensor(flat, parts, group=self.group)
        gathered = flat.view(self.world, 2, max(nc, 1))
        lse_all = gathered[:, 0, :nc].contiguous()
        zy_all = gathered[:, 1, :nc].contiguous()
        self.ops.shard_combine(batch, self.total, self.world, lse_all, zy_all, seq_logp, tok_logp,
                               lse_state, ws, ws_bytes=ws_bytes, stream=stream)

    def backward(self, batch, lse_state, row_coef, dH, dW_shard, accumulate_dW, ws,
                 ws_bytes=None, stream=None):
        """This rank's dW rows; dH summed over the ranks (in place)."""
        import torch.distributed as dist
        self.ops.shard_backward(batch, self.offset, self.total, lse_state, row_coef, dH, dW_shard,
                                accumulate_dW, ws, ws_bytes=ws_bytes, stream=stream)
        if dH is not None:
            dist.all_reduce(dH, group=self.group)
