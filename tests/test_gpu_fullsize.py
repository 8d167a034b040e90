"""CUDA path vs the oracle at the full workload sizes, through the C ABI, in the
launch configuration bench.py times (default workspace, persistent CTA-pair grids).

Every output is compared with the oracle, element by element, at every size:

- "small" (16 rows, d 2048, V 32,000), "llama8b" (the Llama-3.1-8B head: 8 rows of
  2,048 positions, d 4096, V 128,256) and "long" (4 rows of 4,096, d 2048, V 151,936):
  every token log-prob of the policy and the reference forward, every log-sum-exp,
  every row sum, the loss end to end (the GPU's sums through the GPU's loss, against
  the oracle's whole pipeline), margins and accuracy; then the backward fed the loss's
  row coefficients: the whole dH and dW against oracle.backward (relative Frobenius
  error), and also every 256-row vocabulary tile of dW and every scored row of dH on
  its own, so an error confined to a few tiles or rows cannot hide in the global norm.
- "offline" (128 rows of 1,024, d 4096, V 128,256; forward only, want_grad = 0): every
  token log-prob and all 128 row sums.

The oracle's full passes are fp64 matrix products on the host (about 10-100 TFLOP
per configuration); each configuration's results are computed once per module and
reduced to the error figures the tests check, so host memory stays bounded.
"""
import gc

import numpy as np
import pytest

from oracle import dpo_oracle as O
from preference_alignment_b200 import libdpo
from preference_alignment_b200 import workloads as WL

from dpo_harness import (DeviceWorkload, TOL_GRAD, TOL_LOSS, TOL_SEQ_ABS, TOL_SEQ_REL, TOL_TOK,
                         np64, rel_frob)

pytestmark = pytest.mark.gpu

_CACHE = {}
TILE = 256          # vocabulary rows per tile of the dW GEMM


def _seq_errors(gpu, ref):
    err = np.abs(np.asarray(gpu, np.float64) - ref)
    return float(err.max()), float((err / np.maximum(np.abs(ref), 1.0)).max())


def _tile_rel_errors(g, o, tile=TILE, block=8192):
    """Relative Frobenius error of every `tile`-row block of g (fp32) against o (fp64),
    and of the whole array, computed block by block (no full-size temporaries)."""
    n = o.shape[0]
    e2 = np.empty(n)
    r2 = np.empty(n)
    for a in range(0, n, block):
        b = min(n, a + block)
        d = g[a:b].astype(np.float64) - o[a:b]
        e2[a:b] = np.einsum("ij,ij->i", d, d)
        r2[a:b] = np.einsum("ij,ij->i", o[a:b], o[a:b])
    nt = (n + tile - 1) // tile
    te = np.add.reduceat(e2, np.arange(0, nt * tile, tile)[:nt])
    tr = np.add.reduceat(r2, np.arange(0, nt * tile, tile)[:nt])
    whole = float(np.sqrt(e2.sum() / r2.sum()))
    return whole, np.sqrt(te / np.maximum(tr, 1e-300))


def _run(name):
    """GPU and oracle results of one configuration, reduced to error figures."""
    if name in _CACHE:
        return _CACHE[name]
    import torch
    w = WL.make_config(name)
    backward = w.W_ref is not None
    dw = DeviceWorkload(w)
    res = {"w": w, "backward": backward}

    seq, tok, lse = dw.forward(dw.W, want_grad=backward)
    if backward:
        ref, tokr, _ = dw.forward(dw.W_ref, want_grad=False)
    assert libdpo.check() == libdpo.OK
    g_seq, g_tok = np64(seq), np64(tok)

    H64 = WL.widen(w.H, w.dtype)
    W64 = WL.widen(w.W, w.dtype)
    op = O.seq_logprobs(H64, W64, w.tokens, w.prompt_len, w.completion_len)
    res["tok_err"] = float(np.abs(g_tok - op["tok_logp"]).max())
    res["seq_err"] = _seq_errors(g_seq, op["seq_logp"])
    res["n_rows"] = len(g_seq)
    if not backward:
        _CACHE[name] = res
        print(f"\n{name}: " + ", ".join(f"{k} {v}" for k, v in res.items() if k not in ("w",)))
        return res

    res["lse_err"] = float(np.abs(np64(lse)[:w.n_scored] - op["lse"]).max())
    Wr64 = WL.widen(w.W_ref, w.dtype)
    orf = O.seq_logprobs(H64, Wr64, w.tokens, w.prompt_len, w.completion_len)
    del Wr64
    gc.collect()
    res["ref_tok_err"] = float(np.abs(np64(tokr) - orf["tok_logp"]).max())
    res["ref_seq_err"] = _seq_errors(np64(ref), orf["seq_logp"])

    # end to end: GPU sums -> GPU loss, against the oracle's whole pipeline
    ol = O.dpo_loss(op["seq_logp"], orf["seq_logp"], w.beta, w.layout)
    out = dw.loss(seq, ref)
    res["loss"] = (out["loss"].item(), ol["loss"])
    res["margin_err"] = float(np.abs(np64(out["margins"]) - ol["margins"]).max())
    res["accuracy"] = (out["accuracy"].item(), ol["accuracy"])

    # backward with the loss's row coefficients
    coef = torch.from_numpy(ol["row_coef"].astype(np.float32)).cuda()
    dH, dW = dw.backward(lse, coef)
    assert libdpo.check() == libdpo.OK
    gH = dH.cpu().numpy()
    gW = dW.cpu().numpy()
    del dH, dW, dw, seq, tok, lse, ref, tokr, out
    torch.cuda.empty_cache()
    oH, oW = O.backward(H64, W64, w.tokens, w.prompt_len, w.completion_len, ol["row_coef"])
    del W64
    gc.collect()
    res["dW_rel"], tiles = _tile_rel_errors(gW, oW)
    res["dW_tile_rel_max"] = float(tiles.max())
    del gW, oW
    gc.collect()
    pos = O.scored_positions(w.prompt_len, w.completion_len, w.L)
    rows = np.array([p[0] for p in pos])
    ts = np.array([p[1] for p in pos])
    mask = np.ones((w.R, w.L), bool)
    mask[rows, ts] = False
    res["dH_off_completion_zero"] = bool(np.all(gH[mask] == 0.0))
    res["dH_rel"], per_row = _tile_rel_errors(gH[rows, ts], oH[rows, ts], tile=1)
    res["dH_row_rel_max"] = float(per_row.max())
    del gH, oH, H64
    gc.collect()
    _CACHE[name] = res
    print(f"\n{name}: " + ", ".join(f"{k} {v}" for k, v in res.items() if k not in ("w",)))
    return res


# ---------------------------------------------------------------------- small: arrays
def test_small_config_full_parity():
    import torch
    w = WL.make_config("small")
    dw = DeviceWorkload(w)
    H64 = WL.widen(w.H, "bf16")
    W64 = WL.widen(w.W, "bf16")
    Wr64 = WL.widen(w.W_ref, "bf16")
    op = O.seq_logprobs(H64, W64, w.tokens, w.prompt_len, w.completion_len)
    orf = O.seq_logprobs(H64, Wr64, w.tokens, w.prompt_len, w.completion_len)
    ol = O.dpo_loss(op["seq_logp"], orf["seq_logp"], w.beta, w.layout)

    pol, tok, lse = dw.forward(dw.W, want_grad=True)
    ref, tokr, _ = dw.forward(dw.W_ref, want_grad=False)
    out = dw.loss(pol, ref)
    assert libdpo.check() == libdpo.OK
    assert np.abs(np64(tok) - op["tok_logp"]).max() <= TOL_TOK
    assert np.abs(np64(tokr) - orf["tok_logp"]).max() <= TOL_TOK
    assert np.abs(np64(lse)[:w.n_scored] - op["lse"]).max() <= TOL_TOK
    for g, o in ((pol, op), (ref, orf)):
        a, r = _seq_errors(np64(g), o["seq_logp"])
        assert a <= TOL_SEQ_ABS and r <= TOL_SEQ_REL
    assert abs(out["loss"].item() - ol["loss"]) <= TOL_LOSS          # end to end
    np.testing.assert_allclose(np64(out["margins"]), ol["margins"], atol=5e-3)
    assert out["accuracy"].item() == pytest.approx(ol["accuracy"], abs=1e-7)

    dH, dW = dw.backward(lse, torch.from_numpy(ol["row_coef"].astype(np.float32)).cuda())
    assert libdpo.check() == libdpo.OK
    oH, oW = O.backward(H64, W64, w.tokens, w.prompt_len, w.completion_len, ol["row_coef"])
    assert rel_frob(np64(dH), oH) <= TOL_GRAD
    whole, tiles = _tile_rel_errors(dW.cpu().numpy(), oW)
    assert whole <= TOL_GRAD and tiles.max() <= TOL_GRAD


# ---------------------------------------------------------------------- full size
FWD_BWD = ["llama8b", "long"]


@pytest.mark.parametrize("name", FWD_BWD + ["offline"])
def test_every_token_logprob(name):
    r = _run(name)
    assert r["tok_err"] <= TOL_TOK, r["tok_err"]
    if r["backward"]:
        assert r["ref_tok_err"] <= TOL_TOK, r["ref_tok_err"]


@pytest.mark.parametrize("name", FWD_BWD + ["offline"])
def test_every_row_sum(name):
    r = _run(name)
    a, rel = r["seq_err"]
    assert a <= TOL_SEQ_ABS and rel <= TOL_SEQ_REL, r["seq_err"]
    if r["backward"]:
        a, rel = r["ref_seq_err"]
        assert a <= TOL_SEQ_ABS and rel <= TOL_SEQ_REL, r["ref_seq_err"]
    assert r["n_rows"] == r["w"].R


@pytest.mark.parametrize("name", FWD_BWD)
def test_every_logsumexp(name):
    r = _run(name)
    assert r["lse_err"] <= TOL_TOK, r["lse_err"]


@pytest.mark.parametrize("name", FWD_BWD)
def test_loss_end_to_end(name):
    r = _run(name)
    g, o = r["loss"]
    assert abs(g - o) <= TOL_LOSS, (g, o)
    assert r["margin_err"] <= 5e-3
    assert r["accuracy"][0] == pytest.approx(r["accuracy"][1], abs=1e-7)


@pytest.mark.parametrize("name", FWD_BWD)
def test_full_dW_against_the_oracle(name):
    r = _run(name)
    assert r["dW_rel"] <= TOL_GRAD, r["dW_rel"]
    assert r["dW_tile_rel_max"] <= TOL_GRAD, r["dW_tile_rel_max"]


@pytest.mark.parametrize("name", FWD_BWD)
def test_full_dH_against_the_oracle(name):
    r = _run(name)
    assert r["dH_off_completion_zero"]
    assert r["dH_rel"] <= TOL_GRAD, r["dH_rel"]
    assert r["dH_row_rel_max"] <= TOL_GRAD, r["dH_row_rel_max"]
