"""The vocabulary-parallel exchange (preference_alignment_b200.vp) on two CPU ranks (gloo).

Each rank holds one shard of W's rows (vp.shard_range) and the same batch. The
per-shard computations are CPU stand-ins written here from the definitions (the
CUDA entry points need a GPU; their parity is tested on the GPU); what this test
checks is the orchestration: the all-gather of the parts in shard order, the merge
every rank makes, and the dH all-reduce. The result must equal the oracle's
unsharded log-probs and gradients.
"""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import dpo_oracle as O
from preference_alignment_b200 import workloads as WL

WORLD = 2


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _workload():
    return WL.make_custom(R=4, L=30, d=8, V=50, dtype="f32", seed=81, prompt_range=(1, 10),
                          min_completion=2)


class _Batch:
    """What the vp layer passes through: the arrays and the scored-position count."""

    def __init__(self, H, W, tokens, P, C):
        self.H, self.W, self.tokens, self.P, self.C = H, W, tokens, P, C

    @property
    def n_scored(self):
        return int(self.C.sum())

    def scored(self):
        pos = O.scored_positions(self.P, self.C, self.H.shape[1])
        rows = np.array([r for r, _ in pos])
        ts = np.array([t for _, t in pos])
        return rows, ts, self.H[rows, ts], self.tokens[rows, ts + 1]


def _lse(z):
    m = z.max(axis=1, keepdims=True)
    return (m + np.log(np.exp(z - m).sum(axis=1, keepdims=True)))[:, 0]


class CpuShardOps:
    """CPU stand-ins for the three shard entry points (float64 inside)."""

    @staticmethod
    def shard_logprob_parts(b, offset, total, lse_out, zy_out, ws, ws_bytes=None, stream=None):
        _, _, h, y = b.scored()
        z = h @ b.W.T
        here = (y >= offset) & (y < offset + b.W.shape[0])
        zy = np.full(len(y), -np.inf)
        zy[here] = z[np.arange(len(y))[here], (y - offset)[here]]
        lse_out.copy_(torch.from_numpy(_lse(z)))
        zy_out.copy_(torch.from_numpy(zy))

    @staticmethod
    def shard_combine(b, total, n, lse_all, zy_all, seq, tok, lse_state, ws, ws_bytes=None,
                      stream=None):
        rows, ts, _, _ = b.scored()
        parts = lse_all.double().numpy()                 # [n, Nc], shard order
        lse = _lse(parts.T)
        lp = zy_all.double().numpy().max(axis=0) - lse
        t = np.zeros(tok.shape)
        t[rows, ts] = lp
        tok.copy_(torch.from_numpy(t))
        seq.copy_(torch.from_numpy(t.sum(axis=1)))
        lse_state.copy_(torch.from_numpy(lse))

    @staticmethod
    def shard_backward(b, offset, total, lse_state, coef, dH, dW, acc, ws, ws_bytes=None,
                       stream=None):
        rows, ts, h, y = b.scored()
        z = h @ b.W.T
        dz = -np.exp(z - lse_state.double().numpy()[:, None])
        here = (y >= offset) & (y < offset + b.W.shape[0])
        dz[np.arange(len(y))[here], (y - offset)[here]] += 1.0
        dz *= coef.double().numpy()[rows][:, None]
        out = np.zeros(dH.shape)
        out[rows, ts] = dz @ b.W
        dH.copy_(torch.from_numpy(out))
        dW.copy_(torch.from_numpy(dz.T @ h))


def _worker(rank, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=WORLD)
    try:
        from preference_alignment_b200 import vp
        w = _workload()
        H, W = WL.widen(w.H, "f32"), WL.widen(w.W, "f32")
        off, n = vp.shard_range(w.V, WORLD, rank)
        b = _Batch(H, W[off:off + n], w.tokens, w.prompt_len, w.completion_len)
        head = vp.VocabParallelHead(off, w.V, ops=CpuShardOps())
        seq = torch.empty(w.R, dtype=torch.float64)
        tok = torch.empty(w.R, w.L, dtype=torch.float64)
        lse = torch.empty(b.n_scored, dtype=torch.float64)
        head.seq_logprobs(b, seq, tok, lse, ws=None)
        coef = torch.from_numpy(np.linspace(-0.2, 0.3, w.R))
        dH = torch.empty(w.R, w.L, w.d, dtype=torch.float64)
        dW = torch.empty(n, w.d, dtype=torch.float64)
        head.backward(b, lse, coef, dH, dW, False, ws=None)
        q.put((rank, off, seq.numpy(), tok.numpy(), dH.numpy(), dW.numpy()))
    finally:
        dist.destroy_process_group()


def test_two_rank_vocab_parallel_equals_unsharded_oracle():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, port, q)) for r in range(WORLD)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(WORLD):
        r, off, seq, tok, dH, dW = q.get(timeout=120)
        res[r] = (off, seq, tok, dH, dW)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    w = _workload()
    H, W = WL.widen(w.H, "f32"), WL.widen(w.W, "f32")
    o = O.seq_logprobs(H, W, w.tokens, w.prompt_len, w.completion_len)
    oH, oW = O.backward(H, W, w.tokens, w.prompt_len, w.completion_len,
                        np.linspace(-0.2, 0.3, w.R))
    for r in range(WORLD):                               # every rank ends with the same sums and dH
        _, seq, tok, dH, _ = res[r]
        np.testing.assert_allclose(seq, o["seq_logp"], rtol=1e-9, atol=1e-9)
        np.testing.assert_allclose(tok, o["tok_logp"], rtol=1e-9, atol=1e-9)
        np.testing.assert_allclose(dH, oH, rtol=1e-9, atol=1e-12)
    dW = np.concatenate([res[r][4] for r in range(WORLD)])
    assert res[1][0] == res[0][4].shape[0]               # shards are contiguous, in rank order
    np.testing.assert_allclose(dW, oW, rtol=1e-9, atol=1e-12)


def test_shard_range_partitions_the_vocabulary():
    """Shards are disjoint, in rank order, cover [0, total), are non-empty, and are whole
    256-row tiles (but the last) whenever that leaves every rank a row."""
    from preference_alignment_b200 import vp
    for total in (1, 7, 255, 256, 1000, 32000, 128256, 151936, 1 << 24):
        for world in (1, 2, 3, 4, 7, 8, 64):
            if world > total:
                continue
            parts = [vp.shard_range(total, world, r) for r in range(world)]
            at = 0
            for off, n in parts:
                assert off == at and n >= 1
                at += n
            assert at == total
            per = -(-(-(-total // world)) // 256) * 256
            if per * (world - 1) < total:
                assert all(n % 256 == 0 for _, n in parts[:-1])
