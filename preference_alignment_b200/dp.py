"""Data-parallel exchange of the DPO head step.

Each rank scores its own pairs (both rows of a pair stay on one rank) with the
same weights; ranks may hold different numbers of pairs and tokens. The loss is
the mean over all pairs of all ranks (and the NLL term, when used, the mean over
all chosen completion tokens of all ranks), so:

1. `global_counts` sums the pair and chosen-token counts over the ranks;
2. every rank calls dpo_loss_ex with those totals (pairs_total, nll_tokens_total):
   its loss, accuracy, NLL and row coefficients are then its share of the whole
   batch's values, exact for unequal shards;
3. the backward's one exchange is a sum all-reduce of dW. `backward_exchange`
   forms dW block by block of vocabulary rows (dpo_backward_dw) and starts the
   all-reduce of each finished block while the next one is computed, then forms
   dH, which needs no exchange, while the last block's all-reduce runs;
4. `allreduce_shares` sums the loss shares (one small all-reduce).

dH stays on its rank. This mirrors the data-parallel replicas of the pages'
systems ("Run Distributed Full-Model DPO with PyTorch FSDP", Step 1: every rank
holds part of the global batch and the gradients are summed; Megatron-Bridge PR
6092, the DP replicas of its results), at the LM head.
"""
from __future__ import annotations

# Vocabulary rows per dW block are whole 256-row tiles of the dW GEMM (its M tiles),
# so a block boundary never splits a tile.
ROW_ALIGN = 256


def global_counts(pairs: int, chosen_tokens: int, group=None, device=None):
    """(pairs, chosen completion tokens) summed over the ranks of `group`."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([int(pairs), int(chosen_tokens)], dtype=torch.int64, device=device)
    dist.all_reduce(t, group=group)
    return int(t[0]), int(t[1])


def vocab_buckets(V: int, n_buckets: int, align: int = ROW_ALIGN):
    """Split vocabulary rows [0, V) into at most n_buckets contiguous blocks whose
    boundaries are multiples of `align` (the last block ends at V)."""
    if V < 1 or n_buckets < 1:
        raise ValueError("V and n_buckets must be positive")
    tiles = (V + align - 1) // align
    n = min(n_buckets, tiles)
    edges = [min(V, (tiles * b // n) * align) for b in range(n + 1)]
    return [(edges[b], edges[b + 1]) for b in range(n) if edges[b + 1] > edges[b]]


def bucketed_allreduce(dW, buckets, compute_bucket, group=None):
    """For each block (v0, v1): compute_bucket(v0, v1) fills dW[v0:v1] on the current
    stream, then an asynchronous sum all-reduce of those rows starts (on NCCL it
    waits only for the work already enqueued, so it runs while the next block is
    computed). Returns the pending works; call finish(works) before using dW."""
    import torch.distributed as dist
    works = []
    for v0, v1 in buckets:
        compute_bucket(v0, v1)
        works.append(dist.all_reduce(dW[v0:v1], group=group, async_op=True))
    return works


def finish(works):
    """Make the current stream (NCCL) or the host (gloo) wait for the pending all-reduces."""
    for w in works:
        w.wait()


def allreduce_shares(shares, group=None):
    """Sum per-rank shares (e.g. [loss, accuracy, nll]) in place: the whole batch's values."""
    import torch.distributed as dist
    dist.all_reduce(shares, group=group)
    return shares


def backward_exchange(batch, lse_state, row_coef, dH, dW, ws, n_buckets=8, max_sms=0,
                      group=None):
    """The data-parallel backward on this rank: dz once (dpo_backward with dW = NULL),
    then dW block by block with each block's all-reduce started as soon as it is
    formed, then dH while the last all-reduce runs. max_sms > 0 leaves the other SMs
    free for the collective's kernels. Everything is enqueued on torch's current
    stream, the stream the collectives order against. Returns the pending works
    (finish() them)."""
    from preference_alignment_b200 import libdpo
    libdpo.backward(batch, lse_state, row_coef, None, None, False, ws)
    works = bucketed_allreduce(
        dW, vocab_buckets(int(batch.c.V), n_buckets),
        lambda v0, v1: libdpo.backward_dw(batch, v0, v1, dW, False, ws, max_sms=max_sms),
        group=group)
    if dH is not None:
        libdpo.backward_dh(batch, dH, ws, max_sms=max_sms)
    return works


# ------------------------------------------------------------------ fused reduce-scatter
def scatter_rows_per_rank(V: int, n_ranks: int, align: int = ROW_ALIGN) -> int:
    """Rows of W each rank but the last owns in the fused reduce-scatter: whole `align`-row
    tiles, as even as possible, the last rank owning the rest (at least one row)."""
    if V < n_ranks or n_ranks < 1:
        raise ValueError("need at least one vocabulary row per rank")
    tiles = (V + align - 1) // align
    per = -(-tiles // n_ranks) * align
    while per > align and per * (n_ranks - 1) >= V:
        per -= align
    if per * (n_ranks - 1) >= V:          # fewer tiles than ranks: rows, not tiles
        per = V // n_ranks
    return per


def scatter_rows(V: int, n_ranks: int, q: int, per: int) -> range:
    """The rows of W rank q owns."""
    return range(q * per, V if q == n_ranks - 1 else (q + 1) * per)


class FusedReduceScatter:
    """The data-parallel dW exchange fused into the dW GEMM, as a reduce-scatter.

    Rank q owns rows scatter_rows(V, n, q, per) of dW and holds a receive buffer
    [n, rows_q, d] fp32 with one slot per rank. The buffers are shared between the
    processes with CUDA IPC (each rank maps every other rank's buffer), so each rank's
    dW GEMM stores every finished row of its contribution straight into the owner's
    slot (peer memory over NVLink between GPUs) while the GEMM runs; after a barrier
    each owner adds its slots in rank order (the same bits on every run) and holds its
    rows of the summed dW, as a sharded optimiser ("Run Distributed Full-Model DPO
    with PyTorch FSDP", Step 1) needs.

    barrier: called with no arguments where every rank must have finished the work
    enqueued so far. The default is an all-reduce of one number on the current stream
    (NCCL: the host does not wait); for a process group whose collectives are not
    ordered on the stream (gloo), pass one that synchronizes the device first.
    """

    def __init__(self, V: int, d: int, group=None, device=None, barrier=None):
        import torch
        import torch.distributed as dist
        from preference_alignment_b200 import libdpo
        self.group = group
        self.rank = dist.get_rank(group)
        self.n = dist.get_world_size(group)
        if self.n > libdpo.MAX_SCATTER_RANKS:
            raise ValueError(f"at most {libdpo.MAX_SCATTER_RANKS} ranks")
        self.V, self.d = V, d
        self.per = scatter_rows_per_rank(V, self.n)
        self.rows = scatter_rows(V, self.n, self.rank, self.per)
        dev = device if device is not None else torch.device("cuda", torch.cuda.current_device())
        self.recv = torch.empty(self.n, len(self.rows), d, dtype=torch.float32, device=dev)
        handle, offset = libdpo.ipc_export(self.recv)
        shared = [None] * self.n
        dist.all_gather_object(shared, (handle, offset), group=group)
        self.mapped = []
        self.ptrs = []
        try:
            for q, (h, off) in enumerate(shared):
                if q == self.rank:
                    self.ptrs.append(self.recv.data_ptr())
                else:
                    base = libdpo.ipc_import(h)
                    self.mapped.append(base)
                    self.ptrs.append(base + off)
        except Exception:
            self.close()                    # unmap what was mapped before the failure
            raise
        self._flag = torch.zeros(1, device=dev)
        self.barrier = barrier if barrier is not None else self._stream_barrier

    def _stream_barrier(self):
        import torch.distributed as dist
        dist.all_reduce(self._flag, group=self.group)

    def backward(self, batch, lse_state, row_coef, dH, dW_shard, ws, max_sms=0,
                 accumulate=False):
        """dz (dpo_backward with dW = NULL), this rank's dW rows scattered to their owners,
        dH, then the barrier and the sum of this rank's slots into dW_shard ([rows_q, d];
        added to when accumulate), then a second barrier so that no rank's next scatter
        reaches a buffer whose slots are still being summed."""
        from preference_alignment_b200 import libdpo
        libdpo.backward(batch, lse_state, row_coef, None, None, False, ws)
        libdpo.backward_dw_scatter(batch, self.n, self.rank, self.per, self.ptrs, ws,
                                   max_sms=max_sms)
        if dH is not None:
            libdpo.backward_dh(batch, dH, ws, max_sms=max_sms)
        self.barrier()
        libdpo.dw_reduce_slots(self.recv, self.n, len(self.rows), self.d, dW_shard, accumulate)
        self.barrier()

    def close(self):
        from preference_alignment_b200 import libdpo
        for base in self.mapped:
            libdpo.ipc_close(base)
        self.mapped = []
