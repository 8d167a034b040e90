"""The CUDA path against the oracle on seeded random shapes: rows, positions, hidden size
(any multiple of 8), vocabulary (1 to a few thousand, multiples of 8 or not), ragged
prompts and completions (empty ones included), both element types and both row layouts.
Every case compares every token log-prob, row sum and log-sum-exp, the loss end to end,
and dH and dW through the backward with the loss's row coefficients."""
import numpy as np
import pytest

from oracle import dpo_oracle as O
from preference_alignment_b200 import libdpo
from preference_alignment_b200 import workloads as WL

from dpo_harness import (DeviceWorkload, TOL_GRAD, TOL_LOSS, TOL_TOK, assert_seq_close, np64,
                         rel_frob)

pytestmark = pytest.mark.gpu


def _cases(n=48, seed=20261203):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        B = int(rng.integers(1, 6))
        L = int(rng.integers(2, 700))
        d = 8 * int(rng.integers(1, 66))
        special = int(rng.choice([1, 3, 8, 255, 256, 257]))
        V = special if rng.random() < 0.4 else int(rng.integers(2, 5000))
        dtype = "f32" if i % 4 == 3 else "bf16"
        layout = "adjacent" if i % 2 else "halves"
        out.append((2 * B, L, d, V, dtype, layout, int(rng.integers(1, 1 << 30))))
    return out


@pytest.mark.parametrize("R,L,d,V,dtype,layout,seed", _cases())
def test_random_shape_against_the_oracle(R, L, d, V, dtype, layout, seed):
    import torch
    w = WL.make_custom(R=R, L=L, d=d, V=V, dtype=dtype, layout=layout, seed=seed,
                       ref_std=0.05)
    dw = DeviceWorkload(w)
    H = WL.widen(w.H, dtype)
    Wd = WL.widen(w.W, dtype)
    op = O.seq_logprobs(H, Wd, w.tokens, w.prompt_len, w.completion_len)
    orf = O.seq_logprobs(H, WL.widen(w.W_ref, dtype), w.tokens, w.prompt_len, w.completion_len)
    ol = O.dpo_loss(op["seq_logp"], orf["seq_logp"], w.beta, layout)

    pol, tok, lse = dw.forward(dw.W, want_grad=True)
    ref, _, _ = dw.forward(dw.W_ref, want_grad=False)
    out = dw.loss(pol, ref)
    assert libdpo.check() == libdpo.OK
    assert np.abs(np64(tok) - op["tok_logp"]).max(initial=0.0) <= TOL_TOK
    assert np.abs(np64(lse)[:w.n_scored] - op["lse"]).max(initial=0.0) <= TOL_TOK
    assert_seq_close(np64(pol), op["seq_logp"])
    assert_seq_close(np64(ref), orf["seq_logp"])
    assert abs(out["loss"].item() - ol["loss"]) <= TOL_LOSS

    coef = torch.from_numpy(ol["row_coef"].astype(np.float32)).cuda()
    dH, dW = dw.backward(lse, coef)
    assert libdpo.check() == libdpo.OK
    oH, oW = O.backward(H, Wd, w.tokens, w.prompt_len, w.completion_len, ol["row_coef"])
    assert rel_frob(np64(dH), oH) <= TOL_GRAD
    assert rel_frob(np64(dW), oW) <= TOL_GRAD


@pytest.mark.parametrize("R,L,d,V,dtype,layout,seed", _cases(n=16, seed=20261204))
def test_random_shape_chunked_backward_and_vocab_shards(R, L, d, V, dtype, layout, seed):
    """The same comparison through the smallest backward workspace (token chunks of 128
    whenever there are more scored positions) and through the vocabulary-parallel calls
    over 1 to 4 shards run one after the other."""
    import torch
    from preference_alignment_b200.vp import shard_range
    from test_gpu_vocab_shards import _sharded_backward, _sharded_forward
    w = WL.make_custom(R=R, L=L, d=d, V=V, dtype=dtype, layout=layout, seed=seed,
                       ref_std=0.05)
    dw = DeviceWorkload(w)
    H = WL.widen(w.H, dtype)
    Wd = WL.widen(w.W, dtype)
    op = O.seq_logprobs(H, Wd, w.tokens, w.prompt_len, w.completion_len)
    coef_np = np.random.default_rng(seed).normal(0.0, 0.05, R)
    oH, oW = O.backward(H, Wd, w.tokens, w.prompt_len, w.completion_len, coef_np)
    coef = torch.from_numpy(coef_np.astype(np.float32)).cuda()

    _, _, lse = dw.forward(dw.W, want_grad=True)
    _, _, mn = libdpo.workspace_size(dw.batch())
    dH, dW = dw.backward(lse, coef, ws_bytes=mn)
    assert libdpo.check() == libdpo.OK
    assert rel_frob(np64(dH), oH) <= TOL_GRAD
    assert rel_frob(np64(dW), oW) <= TOL_GRAD

    n = min(V, 1 + seed % 4)
    shards = [shard_range(V, n, k) for k in range(n)]
    seq, tok, lse_s, _, _ = _sharded_forward(dw, shards)
    assert libdpo.check() == libdpo.OK
    assert np.abs(np64(tok) - op["tok_logp"]).max(initial=0.0) <= TOL_TOK
    assert_seq_close(np64(seq), op["seq_logp"])
    dHs, dWs = _sharded_backward(dw, shards, lse_s, coef)
    assert libdpo.check() == libdpo.OK
    assert rel_frob(np64(dHs), oH) <= TOL_GRAD
    assert rel_frob(np64(dWs), oW) <= TOL_GRAD
