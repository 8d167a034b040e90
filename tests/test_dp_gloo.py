"""The data-parallel exchange on two CPU ranks (gloo).

Each rank takes its own pairs of a batch (unequal shares: 3 pairs and 1 pair),
sums the pair and chosen-token counts with dp.global_counts, computes its share
of the loss and its LM-head gradients with the oracle using those totals (the
arithmetic dpo_loss_ex does on the GPU), and the ranks exchange dW block by block
of vocabulary rows with dp.bucketed_allreduce and the loss shares with
dp.allreduce_shares. The result must equal the single-process loss and gradients
of the whole batch, and the bucketed all-reduce must equal a single all-reduce of
the whole dW.
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
PAIRS = {0: [0, 1, 2], 1: [3]}          # unequal shares of the 4 pairs


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _workload():
    # 4 pairs, adjacent layout so that pair i = rows 2i, 2i+1 and ranks take whole pairs
    return WL.make_custom(R=8, L=24, d=8, V=40, dtype="f32", layout="adjacent", seed=41,
                          prompt_range=(1, 10), min_completion=2, ref_std=0.3)


def _rows(pairs):
    return np.array([r for i in pairs for r in (2 * i, 2 * i + 1)])


def _grads(w, rows, loss_kw, pairs_total=None, nll_tokens_total=None):
    H = WL.widen(w.H, "f32")[rows]
    W = WL.widen(w.W, "f32")
    Wr = WL.widen(w.W_ref, "f32")
    tok, P, C = w.tokens[rows], w.prompt_len[rows], w.completion_len[rows]
    pol = O.seq_logprobs(H, W, tok, P, C)["seq_logp"]
    ref = O.seq_logprobs(H, Wr, tok, P, C)["seq_logp"]
    lo = O.dpo_loss(pol, ref, w.beta, "adjacent", completion_len=C, pairs_total=pairs_total,
                    nll_tokens_total=nll_tokens_total, **loss_kw)
    dH, dW = O.backward(H, W, tok, P, C, lo["row_coef"])
    return lo, dH, dW


def _worker(rank, port, loss_kw, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=WORLD)
    try:
        w = _workload()
        rows = _rows(PAIRS[rank])
        chosen = int(w.completion_len[rows][0::2].sum())
        Bg, Ng = DP.global_counts(len(PAIRS[rank]), chosen)
        lo, dH, dW_local = _grads(w, rows, loss_kw, pairs_total=Bg, nll_tokens_total=Ng)
        # dW block by block of vocabulary rows: the stand-in for dpo_backward_dw copies
        # this rank's rows of the oracle's dW into place
        dW = torch.zeros(w.V, w.d, dtype=torch.float64)
        src = torch.from_numpy(dW_local)
        buckets = DP.vocab_buckets(w.V, 3, align=8)

        def compute(v0, v1):
            dW[v0:v1] = src[v0:v1]

        DP.finish(DP.bucketed_allreduce(dW, buckets, compute))
        whole = src.clone()
        dist.all_reduce(whole)                      # one all-reduce of the whole dW
        shares = torch.tensor([lo["loss"], lo["accuracy"], lo["nll"]], dtype=torch.float64)
        DP.allreduce_shares(shares)
        q.put((rank, (Bg, Ng), shares.numpy(), dW.numpy(), whole.numpy(), dH,
               lo["row_coef"]))
    finally:
        dist.destroy_process_group()


def _run(loss_kw):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, port, loss_kw, q)) for r in range(WORLD)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(WORLD):
        item = q.get(timeout=120)
        res[item[0]] = item[1:]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return res


@pytest.mark.parametrize("loss_kw", [dict(), dict(nll_weight=0.5),
                                     dict(normalize=True, nll_weight=0.25)])
def test_unequal_shards_equal_the_global_batch(loss_kw):
    res = _run(loss_kw)
    w = _workload()
    whole_rows = np.arange(w.R)
    lo1, dH1, dW1 = _grads(w, whole_rows, loss_kw)       # one process, all pairs
    assert res[0][0] == (4, int(w.completion_len[0::2].sum()))
    for r in range(WORLD):
        counts, shares, dW, dW_whole, dH, coef = res[r]
        assert shares[0] == pytest.approx(lo1["loss"], rel=1e-12)
        assert shares[1] == pytest.approx(lo1["accuracy"], abs=1e-15)
        assert shares[2] == pytest.approx(lo1["nll"], rel=1e-12, abs=1e-15)
        np.testing.assert_allclose(dW, dW1, rtol=1e-10, atol=1e-14)
        rows = _rows(PAIRS[r])
        np.testing.assert_allclose(coef, lo1["row_coef"][rows], rtol=1e-12, atol=1e-18)
        np.testing.assert_allclose(dH, dH1[rows], rtol=1e-10, atol=1e-14)
        # bucketed and whole all-reduce add the same two numbers per element
        assert np.array_equal(dW, dW_whole)


def test_vocab_buckets_tile_aligned_and_covering():
    for V, n in [(128256, 8), (1000, 3), (300, 8), (256, 4), (1, 1), (151936, 5)]:
        b = DP.vocab_buckets(V, n)
        assert b[0][0] == 0 and b[-1][1] == V
        assert all(x[1] == y[0] for x, y in zip(b, b[1:]))
        assert all(v0 % 256 == 0 for v0, _ in b)
        assert all(v1 > v0 for v0, v1 in b)
        assert len(b) <= n
    assert len(DP.vocab_buckets(128256, 8)) == 8
    with pytest.raises(ValueError):
        DP.vocab_buckets(0, 2)


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


def test_scatter_rows_partition_the_vocabulary():
    for V, n in [(128256, 8), (1000, 3), (300, 4), (256, 2), (5, 4), (151936, 8), (70001, 2),
                 (1, 1)]:
        per = DP.scatter_rows_per_rank(V, n)
        rows = [DP.scatter_rows(V, n, q, per) for q in range(n)]
        assert rows[0].start == 0 and rows[-1].stop == V
        assert all(a.stop == b.start for a, b in zip(rows, rows[1:]))
        assert all(len(r) > 0 for r in rows)
        assert all(len(r) == per for r in rows[:-1])
        if V >= 256 * n:
            assert per % 256 == 0                    # whole tiles of the dW GEMM
    with pytest.raises(ValueError):
        DP.scatter_rows_per_rank(3, 4)
