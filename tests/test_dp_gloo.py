"""The data-parallel exchange on two CPU ranks (gloo).

Each rank takes its own pairs of a batch, computes its LM-head gradients with
the oracle using the per-rank grad_scale of preference_alignment_b200.dp, and
the ranks exchange them with dp.allreduce_step. The result must equal the
gradient of the global mean loss over all pairs computed in one process.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import dpo_oracle as O
from preference_alignment_b200 import dp as DP
from preference_alignment_b200 import workloads as WL

WORLD = 2


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _workload():
    # 4 pairs, adjacent layout so that pair i = rows 2i, 2i+1 and ranks take whole pairs
    w = WL.make_custom(R=8, L=24, d=8, V=40, dtype="f32", layout="adjacent", seed=41,
                       prompt_range=(1, 10), min_completion=2, ref_std=0.3)
    return w


def _rank_grads(w, rows, world):
    H = WL.widen(w.H, "f32")[rows]
    W = WL.widen(w.W, "f32")
    Wr = WL.widen(w.W_ref, "f32")
    tok, P, C = w.tokens[rows], w.prompt_len[rows], w.completion_len[rows]
    pol = O.seq_logprobs(H, W, tok, P, C)["seq_logp"]
    ref = O.seq_logprobs(H, Wr, tok, P, C)["seq_logp"]
    lo = O.dpo_loss(pol, ref, w.beta, "adjacent", grad_scale=DP.grad_scale(world))
    dH, dW = O.backward(H, W, tok, P, C, lo["row_coef"])
    return lo["loss"], dH, dW


def _worker(rank, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=WORLD)
    try:
        w = _workload()
        rows = np.arange(4 * rank, 4 * rank + 4)          # pairs 2*rank and 2*rank + 1
        loss, dH, dW = _rank_grads(w, rows, WORLD)
        dW_t = torch.from_numpy(dW)
        loss_t = torch.tensor([loss], dtype=torch.float64)
        DP.allreduce_step(dW_t, loss_t)
        q.put((rank, float(loss_t.item()), dW_t.numpy(), dH))
    finally:
        dist.destroy_process_group()


def test_two_rank_exchange_equals_global_batch():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, port, q)) for r in range(WORLD)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(WORLD):
        r, loss, dW, dH = q.get(timeout=120)
        res[r] = (loss, dW, dH)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    w = _workload()
    loss1, dH1, dW1 = _rank_grads(w, np.arange(8), 1)     # one process, all pairs
    for r in range(WORLD):
        loss, dW, dH = res[r]
        assert loss == pytest.approx(loss1, rel=1e-12)
        np.testing.assert_allclose(dW, dW1, rtol=1e-10, atol=1e-14)
        np.testing.assert_allclose(dH, dH1[4 * r:4 * r + 4], rtol=1e-10, atol=1e-14)


def test_bench_ranks_share_weights_and_not_batches():
    import bench
    a = bench.rank_workload("tiny", 0)
    b = bench.rank_workload("tiny", 1)
    assert np.array_equal(a.W, b.W) and np.array_equal(a.W_ref, b.W_ref)
    assert a.H.dtype == b.H.dtype and a.H.shape == b.H.shape
    assert not np.array_equal(a.H, b.H)
    c = bench.rank_workload("small", 1)
    assert c.H.dtype == np.uint16
    assert np.all(b.prompt_len + b.completion_len <= b.L) and np.all(b.prompt_len >= 1)


def test_rank_batch_without_weights_matches_full_draw():
    import bench
    full = bench.rank_workload("tiny", 1, weights=True)
    light = bench.rank_workload("tiny", 1, weights=False)
    assert light.W is None and light.W_ref is None
    for k in ("prompt_len", "completion_len", "tokens", "H"):
        assert np.array_equal(getattr(full, k), getattr(light, k))
