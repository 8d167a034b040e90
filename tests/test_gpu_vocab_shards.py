"""Vocabulary-parallel head (dpo_shard_logprob_parts / dpo_shard_combine /
dpo_shard_backward) against the oracle, through the C ABI.

The shards of one head are run one after the other on one GPU, and the exchanges
the ranks would make are done here with torch (stacking the per-shard parts as the
all-gather would, summing the partial dH as the all-reduce would). No kernel waits
on another, so one GPU stands in for all ranks.
"""
import numpy as np
import pytest

from oracle import dpo_oracle as O
from preference_alignment_b200 import libdpo
from preference_alignment_b200 import workloads as WL
from preference_alignment_b200.vp import shard_range

from dpo_harness import (DeviceWorkload, TOL_GRAD, TOL_TOK, assert_seq_close, np64, rel_frob)

pytestmark = pytest.mark.gpu


def _shard_batch(dw, o, n, tokens=None):
    w = dw.w
    return libdpo.BatchArgs(dw.H, dw.W[o:o + n], dw.tokens if tokens is None else tokens,
                            w.prompt_len, w.completion_len, dtype=w.dtype)


def _sharded_forward(dw, shards, want_grad=True, tokens=None):
    """Parts of every shard, then the merge. Returns (seq, tok, lse, lse_parts, zy_parts)."""
    import torch
    w = dw.w
    nc = w.n_scored
    lse_parts = torch.empty(len(shards), nc, device="cuda")
    zy_parts = torch.empty(len(shards), nc, device="cuda")
    for k, (o, n) in enumerate(shards):
        b = _shard_batch(dw, o, n, tokens)
        f, _, _ = libdpo.workspace_size(b)
        libdpo.shard_logprob_parts(b, o, w.V, lse_parts[k], zy_parts[k], dw.workspace(f))
    b0 = _shard_batch(dw, *shards[0], tokens)
    f, _, _ = libdpo.workspace_size(b0)
    seq = torch.full((w.R,), float("nan"), device="cuda")
    tok = torch.full((w.R, w.L), float("nan"), device="cuda")
    lse = torch.full((nc,), float("nan"), device="cuda") if want_grad else None
    libdpo.shard_combine(b0, w.V, len(shards), lse_parts, zy_parts, seq, tok, lse, dw.workspace(f))
    return seq, tok, lse, lse_parts, zy_parts


def _sharded_backward(dw, shards, lse, coef, tokens=None):
    """dH = sum of the shards' partial dH (the all-reduce), dW = the shards' rows stacked."""
    import torch
    w = dw.w
    dH = torch.zeros(w.R, w.L, w.d, device="cuda", dtype=torch.float64)
    dWs = []
    for o, n in shards:
        b = _shard_batch(dw, o, n, tokens)
        _, bw, _ = libdpo.workspace_size(b)
        part = torch.full((w.R, w.L, w.d), float("nan"), device="cuda")
        dWk = torch.full((n, w.d), float("nan"), device="cuda")
        libdpo.shard_backward(b, o, w.V, lse, coef, part, dWk, False, dw.workspace(bw))
        dH += part.double()
        dWs.append(dWk)
    return dH, torch.cat(dWs)


SPLITS = {
    "aligned3": None,                                   # shard_range over 3 ranks
    "ragged": [(0, 700), (700, 601), (1301, 1699)],     # offsets off the 256-row tiles
    "tiny_last": [(0, 2999), (2999, 1)],                # a one-row shard
}


@pytest.mark.parametrize("split", sorted(SPLITS))
def test_sharded_forward_and_backward_match_oracle(split):
    import torch
    w = WL.make_custom(R=6, L=200, d=256, V=3000, dtype="bf16", seed=71, prompt_range=(1, 80))
    shards = SPLITS[split] or [shard_range(w.V, 3, k) for k in range(3)]
    dw = DeviceWorkload(w)
    H, W = WL.widen(w.H, "bf16"), WL.widen(w.W, "bf16")
    o = O.seq_logprobs(H, W, w.tokens, w.prompt_len, w.completion_len)
    seq, tok, lse, lse_parts, zy_parts = _sharded_forward(dw, shards)
    assert libdpo.check() == libdpo.OK
    assert np.abs(np64(tok) - o["tok_logp"]).max() <= TOL_TOK
    assert_seq_close(np64(seq), o["seq_logp"])
    assert np.abs(np64(lse) - o["lse"]).max() <= TOL_TOK

    # each shard's parts against the oracle on that shard's rows
    pos = o["positions"]
    rows = np.array([r for r, _ in pos])
    ts = np.array([t for _, t in pos])
    h = H[rows, ts]
    y = w.tokens[rows, ts + 1]
    for k, (off, n) in enumerate(shards):
        here = (y >= off) & (y < off + n)
        lp_k, lse_k = O.position_logprobs(h, W[off:off + n], np.where(here, y - off, 0))
        assert np.abs(np64(lse_parts[k]) - lse_k).max() <= TOL_TOK
        zy = np64(zy_parts[k])
        assert np.all(np.isneginf(zy[~here]))
        if here.any():
            assert np.abs(zy[here] - (lp_k + lse_k)[here]).max() <= TOL_TOK

    coef = np.random.default_rng(72).normal(0, 0.05, size=w.R).astype(np.float32)
    dH, dW = _sharded_backward(dw, shards, lse, torch.from_numpy(coef).cuda())
    assert libdpo.check() == libdpo.OK
    oH, oW = O.backward(H, W, w.tokens, w.prompt_len, w.completion_len, coef.astype(np.float64))
    assert rel_frob(np64(dH), oH) <= TOL_GRAD
    assert rel_frob(np64(dW), oW) <= TOL_GRAD


def test_one_shard_is_the_unsharded_path_bit_for_bit():
    import torch
    w = WL.make_custom(R=4, L=300, d=256, V=2000, dtype="bf16", seed=73, prompt_range=(1, 100))
    dw = DeviceWorkload(w)
    seq, tok, lse, _, _ = _sharded_forward(dw, [(0, w.V)])
    seq1, tok1, lse1 = dw.forward(dw.W, want_grad=True)
    assert torch.equal(seq, seq1) and torch.equal(tok, tok1) and torch.equal(lse, lse1)
    coef = torch.linspace(-0.1, 0.1, w.R, device="cuda")
    b = _shard_batch(dw, 0, w.V)
    _, bw, _ = libdpo.workspace_size(b)
    dH = torch.empty(w.R, w.L, w.d, device="cuda")
    dW = torch.empty(w.V, w.d, device="cuda")
    libdpo.shard_backward(b, 0, w.V, lse, coef, dH, dW, False, dw.workspace(bw))
    dH1, dW1 = dw.backward(lse1, coef)
    assert libdpo.check() == libdpo.OK
    assert torch.equal(dH, dH1) and torch.equal(dW, dW1)


def test_fp32_tiny_config_in_two_shards():
    import torch
    w = WL.make_config("tiny")
    dw = DeviceWorkload(w)
    shards = [(0, 400), (400, 600)]
    H, W = WL.widen(w.H, w.dtype), WL.widen(w.W, w.dtype)
    o = O.seq_logprobs(H, W, w.tokens, w.prompt_len, w.completion_len)
    seq, tok, lse, _, _ = _sharded_forward(dw, shards)
    assert np.abs(np64(tok) - o["tok_logp"]).max() <= TOL_TOK
    assert_seq_close(np64(seq), o["seq_logp"])
    coef = np.random.default_rng(74).normal(0, 0.05, size=w.R).astype(np.float32)
    dH, dW = _sharded_backward(dw, shards, lse, torch.from_numpy(coef).cuda())
    assert libdpo.check() == libdpo.OK
    oH, oW = O.backward(H, W, w.tokens, w.prompt_len, w.completion_len, coef.astype(np.float64))
    assert rel_frob(np64(dH), oH) <= TOL_GRAD
    assert rel_frob(np64(dW), oW) <= TOL_GRAD


def test_bad_targets_in_shards():
    """A token outside [0, V) scores 0 and gets no gradient, as in the unsharded path."""
    import torch
    w = WL.make_custom(R=4, L=120, d=128, V=1500, dtype="bf16", seed=75, prompt_range=(1, 40))
    w.prompt_len[1], w.completion_len[1] = 20, 50
    dw = DeviceWorkload(w)
    toks = w.tokens.copy()
    r, p = 1, int(w.prompt_len[1])
    toks[r, p + 2] = w.V + 5                   # the third completion token of row 1
    tdev = torch.from_numpy(toks).cuda()
    shards = [(0, 512), (512, 988)]
    seq, tok, lse, _, _ = _sharded_forward(dw, shards, tokens=tdev)
    assert libdpo.check() == libdpo.ERR_BAD_TARGET
    ref_b = libdpo.BatchArgs(dw.H, dw.W, tdev, w.prompt_len, w.completion_len, dtype="bf16")
    seq1, tok1, lse1 = dw.forward(want_grad=True, batch=ref_b)
    assert libdpo.check() == libdpo.ERR_BAD_TARGET
    t = np64(tok)
    assert t[r, p + 1] == 0.0
    assert np.abs(t - np64(tok1)).max() <= 1e-5
    coef = torch.full((w.R,), 0.05, device="cuda")
    dH, dW = _sharded_backward(dw, shards, lse, coef, tokens=tdev)
    dH1, dW1 = dw.backward(lse1, coef, batch=ref_b)
    assert libdpo.check() == libdpo.ERR_BAD_TARGET
    assert np.all(np64(dH)[r, p + 1] == 0.0)
    assert rel_frob(np64(dH), np64(dH1)) <= 1e-3
    assert rel_frob(np64(dW), np64(dW1)) <= 1e-3


def test_llama8b_head_in_eight_shards():
    """Full size: the 8-shard result equals the unsharded path's within fp32 rounding
    (the unsharded path is checked against the oracle at this size elsewhere)."""
    import torch
    w = WL.make_config("llama8b", with_ref=False)
    dw = DeviceWorkload(w)
    shards = [shard_range(w.V, 8, k) for k in range(8)]
    seq, tok, lse, _, _ = _sharded_forward(dw, shards)
    seq1, tok1, lse1 = dw.forward(dw.W, want_grad=True)
    assert libdpo.check() == libdpo.OK
    assert (lse - lse1).abs().max().item() <= 1e-4
    assert (tok - tok1).abs().max().item() <= 1e-4
    assert (seq.double() - seq1.double()).abs().max().item() <= 5e-2
    coef = torch.linspace(-0.02, 0.02, w.R, device="cuda")
    dH, dW = _sharded_backward(dw, shards, lse1, coef)
    dH1, dW1 = dw.backward(lse1, coef)
    assert libdpo.check() == libdpo.OK
    assert rel_frob(np64(dH), np64(dH1)) <= 1e-3
    assert rel_frob(np64(dW), np64(dW1)) <= 1e-3


def test_shard_calls_and_logits_mean_replay_from_a_cuda_graph():
    """Two shards' parts, the merge, both shard backwards and the logits mean, captured
    into one CUDA graph and replayed: the same outputs as the direct calls."""
    import torch
    w = WL.make_custom(R=4, L=160, d=256, V=1300, dtype="bf16", seed=76, prompt_range=(1, 60))
    dw = DeviceWorkload(w)
    shards = [(0, 768), (768, 532)]
    nc = w.n_scored
    bs = [_shard_batch(dw, o, n) for o, n in shards]
    need = max(max(libdpo.workspace_size(b)[:2]) for b in bs)
    wss = [dw.workspace(need) for _ in shards]
    parts = torch.empty(2, len(shards), nc, device="cuda")
    seq = torch.empty(w.R, device="cuda")
    lse = torch.empty(nc, device="cuda")
    coef = torch.linspace(-0.1, 0.1, w.R, device="cuda")
    dHs = [torch.empty(w.R, w.L, w.d, device="cuda") for _ in shards]
    dWs = [torch.empty(n, w.d, device="cuda") for _, n in shards]
    means = torch.empty(2, device="cuda")
    full = libdpo.BatchArgs(dw.H, dw.W, dw.tokens, w.prompt_len, w.completion_len, dtype="bf16")
    ws_full = dw.workspace(libdpo.workspace_size(full)[0])

    def run(stream):
        for k, ((o, n), b) in enumerate(zip(shards, bs)):
            libdpo.shard_logprob_parts(b, o, w.V, parts[0, k], parts[1, k], wss[k], stream=stream)
        libdpo.shard_combine(bs[0], w.V, len(shards), parts[0], parts[1], seq, None, lse, wss[0],
                             stream=stream)
        for k, ((o, n), b) in enumerate(zip(shards, bs)):
            libdpo.shard_backward(b, o, w.V, lse, coef, dHs[k], dWs[k], False, wss[k],
                                  stream=stream)
        libdpo.logits_mean(full, "halves", means, ws_full, stream=stream)

    outs = [parts, seq, lse, *dHs, *dWs, means]
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        run(s.cuda_stream)
    s.synchronize()
    direct = [t.clone() for t in outs]
    for t in outs:
        t.fill_(float("nan"))
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        run(s.cuda_stream)
    g.replay()
    torch.cuda.synchronize()
    assert libdpo.check() == libdpo.OK
    for a, b in zip(direct, outs):
        assert torch.equal(a, b)
