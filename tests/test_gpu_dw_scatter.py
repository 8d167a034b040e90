"""The data-parallel dW exchange fused into the dW GEMM (a reduce-scatter over
receive buffers shared between processes with CUDA IPC).

Every rank forms its whole contribution dz_r^T . Hp_r and the GEMM's epilogue stores
each row into the owner rank's buffer, in this rank's slot; each owner then adds its
slots in rank order. The expected result is the separately computed dW of every
rank (the one-call backward, checked against the oracle elsewhere) summed in rank
order in fp32, so the comparison is bit for bit.

On one GPU: (1) several ranks emulated in one process (the "peer" buffers are this
process's own), and (2) two processes on the same GPU sharing their buffers through
CUDA IPC, synchronised by a host barrier (gloo). No kernel ever waits for another.
"""
import os
import socket

import numpy as np
import pytest

from preference_alignment_b200 import dp as DP
from preference_alignment_b200 import libdpo
from preference_alignment_b200 import workloads as WL

from dpo_harness import DeviceWorkload

pytestmark = pytest.mark.gpu

SHAPE = dict(L=300, d=256, V=1000, dtype="bf16", prompt_range=(1, 120), full_rows=1)


def _rank_batch(rank, R=4):
    """Rank `rank`'s batch: its own rows, the shared weights (seed 61)."""
    w = WL.make_custom(R=R, seed=61, **SHAPE)
    own = WL.make_custom(R=R, seed=100 + rank, **SHAPE)
    w.H, w.tokens, w.prompt_len, w.completion_len = own.H, own.tokens, own.prompt_len, own.completion_len
    return w


def _dz_and_dW(w):
    """The rank's forward, coefficients, dz left in a workspace, and its one-call dW."""
    import torch
    dw = DeviceWorkload(w)
    _, _, lse = dw.forward(dw.W, want_grad=True)
    coef = torch.from_numpy(np.random.default_rng(w.seed).normal(0, 0.05, w.R).astype(np.float32)).cuda()
    _, dW = dw.backward(lse, coef, want_dH=False)
    b = dw.batch()
    _, bwd, _ = libdpo.workspace_size(b)
    ws = dw.workspace(bwd)
    libdpo.backward(b, lse, coef, None, None, False, ws)     # dz stays in ws
    return dw, b, ws, dW


@pytest.mark.parametrize("n_ranks", [1, 3])
def test_emulated_ranks_in_one_process(n_ranks):
    import torch
    V, d = SHAPE["V"], SHAPE["d"]
    per = DP.scatter_rows_per_rank(V, n_ranks)
    rows = [DP.scatter_rows(V, n_ranks, q, per) for q in range(n_ranks)]
    recv = [torch.full((n_ranks, len(r), d), float("nan"), device="cuda") for r in rows]
    total = None
    ranks = [_dz_and_dW(_rank_batch(r)) for r in range(n_ranks)]
    for r, (dw, b, ws, dW) in enumerate(ranks):
        libdpo.backward_dw_scatter(b, n_ranks, r, per, recv, ws, max_sms=100)
        total = dW.clone() if total is None else total + dW
    for q in range(n_ranks):
        shard = torch.full((len(rows[q]), d), float("nan"), device="cuda")
        libdpo.dw_reduce_slots(recv[q], n_ranks, len(rows[q]), d, shard)
        assert libdpo.check() == libdpo.OK
        assert torch.equal(shard, total[rows[q].start:rows[q].stop])
        libdpo.dw_reduce_slots(recv[q], n_ranks, len(rows[q]), d, shard, accumulate=True)
        assert torch.equal(shard, 2 * total[rows[q].start:rows[q].stop])


def test_rank_without_scored_positions_sends_zeros():
    import torch
    V, d = SHAPE["V"], SHAPE["d"]
    w = _rank_batch(0)
    w.completion_len = np.zeros_like(w.completion_len)
    dw = DeviceWorkload(w)
    b = dw.batch()
    _, bwd, _ = libdpo.workspace_size(b)
    ws = dw.workspace(bwd)
    lse = torch.empty(1, device="cuda")
    libdpo.backward(b, lse, torch.zeros(w.R, device="cuda"), None, None, False, ws)
    per = DP.scatter_rows_per_rank(V, 2)
    recv = [torch.full((2, len(DP.scatter_rows(V, 2, q, per)), d), 7.0, device="cuda")
            for q in range(2)]
    libdpo.backward_dw_scatter(b, 2, 1, per, recv, ws)
    assert libdpo.check() == libdpo.OK
    for q in range(2):
        assert torch.all(recv[q][1] == 0) and torch.all(recv[q][0] == 7.0)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _ipc_worker(rank, world, port, q):
    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        libdpo.load()

        def host_barrier():
            torch.cuda.synchronize()
            dist.barrier()

        V, d = SHAPE["V"], SHAPE["d"]
        ex = DP.FusedReduceScatter(V, d, barrier=host_barrier)
        dw, b, ws, dW_own = _dz_and_dW(_rank_batch(rank))
        _, _, lse = dw.forward(dw.W, want_grad=True)
        coef = torch.from_numpy(np.random.default_rng(dw.w.seed).normal(0, 0.05, dw.w.R)
                                .astype(np.float32)).cuda()
        shard = torch.full((len(ex.rows), d), float("nan"), device="cuda")
        ex.backward(b, lse, coef, None, shard, ws, max_sms=100)
        torch.cuda.synchronize()
        ok_status = libdpo.check() == libdpo.OK
        # the expected sum: every rank's one-call dW, recomputed here, in rank order
        total = None
        for r in range(world):
            dW_r = dW_own if r == rank else _dz_and_dW(_rank_batch(r))[3]
            total = dW_r.clone() if total is None else total + dW_r
        same = bool(torch.equal(shard, total[ex.rows.start:ex.rows.stop]))
        ex.close()
        dist.barrier()
        q.put((rank, ok_status, same, len(ex.rows)))
    finally:
        dist.destroy_process_group()


def test_two_processes_share_receive_buffers_through_ipc():
    import torch.multiprocessing as mp
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ipc_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        rank, ok_status, same, n_rows = q.get(timeout=300)
        res[rank] = (ok_status, same, n_rows)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert sum(r[2] for r in res.values()) == SHAPE["V"]
    for rank in range(world):
        assert res[rank][0], f"rank {rank}: device status"
        assert res[rank][1], f"rank {rank}: shard differs from the rank-order sum"
