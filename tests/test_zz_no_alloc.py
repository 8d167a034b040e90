"""The workspace-free forward entry point, dpo_seq_logprobs_noalloc.

It serves callers that may not allocate device memory (a framework that owns
the device-memory budget and forbids allocation from its plugins, or code that
cannot accept the synchronisation cudaMalloc/cudaFree may cause). The forward is
deterministic, so its results must equal those of dpo_seq_logprobs, which takes a
caller workspace, bit for bit, call after call (the built-in scratch is shared and
keeps the previous call's contents), and match the oracle within the path's
tolerances. This file is collected last on purpose.
"""
import numpy as np
import pytest

from oracle import dpo_oracle as O
from preference_alignment_b200 import libdpo
from preference_alignment_b200 import workloads as WL

from dpo_harness import DeviceWorkload, TOL_TOK, assert_seq_close, np64

pytestmark = pytest.mark.gpu


def _noalloc(dw):
    import torch
    w = dw.w
    b = dw.batch()
    seq = torch.full((w.R,), float("nan"), device="cuda")
    tok = torch.full((w.R, w.L), float("nan"), device="cuda")
    lse = torch.full((max(w.n_scored, 1),), float("nan"), device="cuda")
    libdpo.seq_logprobs_noalloc(b, True, seq, tok, lse)
    return seq, tok, lse


def test_noalloc_matches_workspace_entry_point_on_consecutive_calls():
    cases = [
        WL.make_custom(R=6, L=300, d=256, V=1000, dtype="bf16", seed=31, prompt_range=(1, 200),
                       full_rows=1),
        WL.make_custom(R=4, L=500, d=512, V=3000, dtype="bf16", seed=32, prompt_range=(1, 100),
                       full_rows=2),
    ]
    import torch
    for k, w in enumerate(cases):
        dw = DeviceWorkload(w)
        fwd, _, _ = libdpo.workspace_size(dw.batch())
        assert fwd <= libdpo.NOALLOC_SCRATCH_BYTES
        seq_a, tok_a, lse_a = dw.forward(dw.W, want_grad=True)     # caller workspace
        seq_b, tok_b, lse_b = _noalloc(dw)                          # built-in scratch
        assert libdpo.check() == libdpo.OK
        nc = w.n_scored
        assert torch.equal(seq_b, seq_a)
        assert torch.equal(tok_b, tok_a)
        assert torch.equal(lse_b[:nc], lse_a[:nc])
        if k == 0:
            o = O.seq_logprobs(WL.widen(w.H, w.dtype), WL.widen(w.W, w.dtype), w.tokens,
                               w.prompt_len, w.completion_len)
            assert np.abs(np64(tok_b) - o["tok_logp"]).max() <= TOL_TOK
            assert_seq_close(np64(seq_b), o["seq_logp"])
            assert np.abs(np64(lse_b)[:nc] - o["lse"]).max() <= TOL_TOK


def test_noalloc_refuses_batches_beyond_its_scratch():
    import torch
    w = WL.make_custom(R=2, L=4096, d=2048, V=32000, dtype="bf16", seed=33, prompt_range=(1, 8),
                       full_rows=2, with_ref=False)
    dw = DeviceWorkload(w)
    fwd, _, _ = libdpo.workspace_size(dw.batch())
    assert fwd > libdpo.NOALLOC_SCRATCH_BYTES
    seq = torch.full((w.R,), 3.0, device="cuda")
    with pytest.raises(libdpo.DpoError) as e:
        libdpo.seq_logprobs_noalloc(dw.batch(), False, seq, None, None)
    assert e.value.status == libdpo.ERR_WORKSPACE
    assert np.all(np64(seq) == 3.0)
