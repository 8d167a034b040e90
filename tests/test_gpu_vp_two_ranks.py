"""The vocabulary-parallel head with the library's kernels on two processes sharing
one GPU (gloo collectives; no kernel waits on another).

Each rank holds one shard of W's rows (vp.shard_range, a ragged split) and the same
batch; vp.VocabParallelHead gathers the shards' parts, merges them and sums the
partial dH. Every rank must then hold the unsharded path's sums, token log-probs and
dH (one process, the whole W), and its shard of the unsharded dW.
"""
import os
import socket

import numpy as np
import pytest

from preference_alignment_b200 import libdpo
from preference_alignment_b200 import vp as VP
from preference_alignment_b200 import workloads as WL

from dpo_harness import DeviceWorkload, TOL_TOK, assert_seq_close, np64, rel_frob

pytestmark = pytest.mark.gpu

V = 2300          # 8 tiles of 256 and a ragged 252-row tail


def _workload():
    return WL.make_custom(R=6, L=260, d=256, V=V, dtype="bf16", seed=63, prompt_range=(1, 90),
                          full_rows=1)


def _worker(rank, world, port, q):
    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        libdpo.load()
        w = _workload()
        dw = DeviceWorkload(w)
        # the unsharded path, for comparison
        seq1, tok1, lse1 = dw.forward(dw.W, want_grad=True)
        coef = torch.linspace(-0.2, 0.3, w.R, device="cuda")
        dH1, dW1 = dw.backward(lse1, coef)
        # this rank's shard
        off, rows = VP.shard_range(V, world, rank)
        Wsh = dw.W[off:off + rows].contiguous()
        b = dw.batch(W=Wsh)
        fwd, bwd, _ = libdpo.workspace_size(b)
        ws = dw.workspace(max(fwd, bwd))
        head = VP.VocabParallelHead(off, V)
        seq = torch.empty(w.R, device="cuda")
        tok = torch.empty(w.R, w.L, device="cuda")
        lse = torch.empty(w.n_scored, device="cuda")
        head.seq_logprobs(b, seq, tok, lse, ws)
        dH = torch.empty(w.R, w.L, w.d, device="cuda")
        dWs = torch.empty(rows, w.d, device="cuda")
        head.backward(b, lse, coef, dH, dWs, False, ws)
        torch.cuda.synchronize()
        q.put((rank, libdpo.check(), float(np.abs(np64(tok) - np64(tok1)).max()),
               np64(seq), np64(seq1), rel_frob(np64(dH), np64(dH1)),
               rel_frob(np64(dWs), np64(dW1[off:off + rows])), rows))
    finally:
        dist.destroy_process_group()


def test_two_ranks_equal_the_unsharded_path():
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
    assert sum(r[7] for r in res) == V
    for rank, status, tok_err, seq, seq1, dH_err, dW_err, _ in res:
        assert status == libdpo.OK
        assert tok_err <= TOL_TOK
        assert_seq_close(seq, seq1)
        assert dH_err <= 1e-3          # partial dH of two shards summed vs one launch
        assert dW_err <= 1e-5          # the shard's rows: the same GEMM over the same rows
