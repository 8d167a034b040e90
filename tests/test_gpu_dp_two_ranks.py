"""The data-parallel step with the library's kernels on two processes sharing one GPU
(gloo collectives; no kernel waits on another).

Rank 0 holds 3 pairs and rank 1 holds 1 pair of a 4-pair batch (adjacent layout). Each
rank sums the pair and chosen-token counts (dp.global_counts), calls dpo_loss_ex with
them (its loss, accuracy, NLL and row coefficients are its share), runs
dp.backward_exchange (dz, dW by blocks of vocabulary rows with an all-reduce per
block, dH) and sums the loss shares. Every rank must then hold the single-process
loss and dW of the whole batch (the same kernels over all four pairs in one process),
and its own rows of dH.
"""
import os
import socket

import numpy as np
import pytest

from preference_alignment_b200 import dp as DP
from preference_alignment_b200 import libdpo
from preference_alignment_b200 import workloads as WL

from dpo_harness import DeviceWorkload, np64, rel_frob

pytestmark = pytest.mark.gpu

PAIRS = {0: [0, 1, 2], 1: [3]}
NLL = 0.3


def _batch():
    return WL.make_custom(R=8, L=240, d=256, V=1500, dtype="bf16", layout="adjacent", seed=62,
                          prompt_range=(1, 100), min_completion=1, ref_std=0.05)


def _subset(w, pairs):
    rows = np.array([r for i in pairs for r in (2 * i, 2 * i + 1)])
    v = WL.make_custom(R=len(rows), L=w.L, d=w.d, V=w.V, dtype=w.dtype, layout=w.layout,
                       seed=w.seed, prompt_range=(1, 2), ref_std=0.05)
    v.W, v.W_ref = w.W, w.W_ref
    v.H, v.tokens = np.ascontiguousarray(w.H[rows]), np.ascontiguousarray(w.tokens[rows])
    v.prompt_len = np.ascontiguousarray(w.prompt_len[rows])
    v.completion_len = np.ascontiguousarray(w.completion_len[rows])
    return v


def _step(w, pairs_total=0, nll_tokens_total=0, exchange=None):
    """Policy and reference forward, loss (shares when the totals are given), backward."""
    import torch
    dw = DeviceWorkload(w)
    pol, _, lse = dw.forward(dw.W, want_grad=True)
    ref, _, _ = dw.forward(dw.W_ref, want_grad=False)
    B = w.R // 2
    out = {k: torch.empty(n, device="cuda") for k, n in
           [("shares", 3), ("coef", 2 * B)]}
    clen = torch.from_numpy(w.completion_len).cuda()
    libdpo.loss_ex(B, w.layout, pol, ref, w.beta, 1.0, out["shares"][0:1], out["shares"][1:2],
                   row_coef=out["coef"], nll=out["shares"][2:3], nll_weight=NLL,
                   completion_len=clen, pairs_total=pairs_total, nll_tokens_total=nll_tokens_total)
    if exchange is None:
        dH, dW = dw.backward(lse, out["coef"])
    else:
        b = dw.batch()
        _, bwd, _ = libdpo.workspace_size(b)
        ws = dw.workspace(bwd)
        dH = torch.empty(w.R, w.L, w.d, device="cuda")
        dW = torch.empty(w.V, w.d, device="cuda")
        exchange(b, lse, out["coef"], dH, dW, ws)
    return out["shares"], dH, dW


def _worker(rank, world, port, q):
    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        libdpo.load()
        w = _batch()
        mine = _subset(w, PAIRS[rank])
        Bg, Ng = DP.global_counts(len(PAIRS[rank]), int(mine.completion_len[0::2].sum()))

        def exchange(b, lse, coef, dH, dW, ws):
            DP.finish(DP.backward_exchange(b, lse, coef, dH, dW, ws, n_buckets=3, max_sms=100))

        shares, dH, dW = _step(mine, Bg, Ng, exchange)
        DP.allreduce_shares(shares)
        torch.cuda.synchronize()
        status = libdpo.check()
        s1, dH1, dW1 = _step(w)                                # one process, all four pairs
        rows = [r for i in PAIRS[rank] for r in (2 * i, 2 * i + 1)]
        q.put((rank, status, np64(shares), np64(s1), rel_frob(np64(dW), np64(dW1)),
               rel_frob(np64(dH), np64(dH1[rows])), (Bg, Ng)))
    finally:
        dist.destroy_process_group()


def test_two_ranks_unequal_shards_equal_one_process():
    import torch.multiprocessing as mp
    world = 2
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=300) for _ in range(world)]
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    w = _batch()
    assert all(r[6] == (4, int(w.completion_len[0::2].sum())) for r in res)
    for rank, status, shares, single, dW_err, dH_err, _ in res:
        assert status == libdpo.OK
        assert shares[0] == pytest.approx(single[0], abs=2e-6)      # loss
        assert shares[1] == pytest.approx(single[1], abs=1e-7)      # accuracy
        assert shares[2] == pytest.approx(single[2], rel=1e-5)      # NLL
        assert dW_err <= 1e-5          # two GEMMs over the ranks' tokens, added, vs one GEMM
        assert dH_err <= 1e-6
