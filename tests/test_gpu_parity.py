"""CUDA path vs the CPU fp64 oracle, element by element, through the C ABI.

Sizes here are small enough for the oracle to finish in seconds while spanning
several 128-position and 256-vocab tiles with ragged tails.
"""
import math

import numpy as np
import pytest

from oracle import dpo_oracle as O
from preference_alignment_b200 import libdpo
from preference_alignment_b200 import workloads as WL

from dpo_harness import (DeviceWorkload, TOL_GRAD, TOL_LOSS, TOL_TOK, assert_seq_close, np64,
                         rel_frob)

pytestmark = pytest.mark.gpu


def _oracle_fwd(w, W):
    H = WL.widen(w.H, w.dtype)
    return O.seq_logprobs(H, WL.widen(W, w.dtype), w.tokens, w.prompt_len, w.completion_len)


def _check_forward(dw, W_np, W_dev):
    w = dw.w
    o = _oracle_fwd(w, W_np)
    seq, tok, lse = dw.forward(W_dev, want_grad=True)
    assert libdpo.check() == libdpo.OK
    tok = np64(tok)
    assert np.all(np.isfinite(tok))
    err = np.abs(tok - o["tok_logp"])
    assert err.max() <= TOL_TOK, f"token lp err {err.max()}"
    assert_seq_close(np64(seq), o["seq_logp"])
    np.testing.assert_allclose(np64(lse)[:len(o["lse"])], o["lse"], rtol=0, atol=TOL_TOK)
    return o, seq, tok, lse


SHAPES = [
    # R, L, d, V, prompt range, seed
    (4, 96, 64, 256, (1, 40), 1),          # one vocab tile, one k block
    (6, 300, 256, 1000, (1, 200), 2),      # ragged vocab tail (1000 = 3*256 + 232)
    (8, 200, 200, 777, (1, 150), 3),       # d not a multiple of 64: K tail zero-filled
    (2, 700, 128, 2048, (1, 100), 4),      # positions span 5+ M tiles with a ragged tail
    (10, 64, 512, 513, (1, 63), 5),        # V = 2*256 + 1: one valid column in the last tile
]


@pytest.mark.parametrize("R,L,d,V,pr,seed", SHAPES)
def test_forward_bf16_small(R, L, d, V, pr, seed):
    w = WL.make_custom(R=R, L=L, d=d, V=V, dtype="bf16", seed=seed, prompt_range=pr, full_rows=1)
    dw = DeviceWorkload(w)
    _check_forward(dw, w.W, dw.W)


def test_forward_f32_tiny_config():
    w = WL.make_config("tiny")
    dw = DeviceWorkload(w)
    _check_forward(dw, w.W, dw.W)


@pytest.mark.parametrize("R,L,d,V,pr,seed", SHAPES[:4])
def test_backward_bf16_small(R, L, d, V, pr, seed):
    w = WL.make_custom(R=R, L=L, d=d, V=V, dtype="bf16", seed=seed, prompt_range=pr, full_rows=1)
    dw = DeviceWorkload(w)
    seq, tok, lse = dw.forward(dw.W, want_grad=True)
    coef = np.random.default_rng(seed).normal(0, 0.05, size=R).astype(np.float32)
    import torch
    coef_dev = torch.from_numpy(coef).cuda()
    dH, dW = dw.backward(lse, coef_dev)
    assert libdpo.check() == libdpo.OK
    H = WL.widen(w.H, "bf16")
    Wd = WL.widen(w.W, "bf16")
    oH, oW = O.backward(H, Wd, w.tokens, w.prompt_len, w.completion_len, coef.astype(np.float64))
    assert rel_frob(np64(dH), oH) <= TOL_GRAD
    assert rel_frob(np64(dW), oW) <= TOL_GRAD
    # unscored positions are exactly zero
    gH = np64(dH)
    for r in range(R):
        p, c = w.prompt_len[r], w.completion_len[r]
        mask = np.ones(L, bool)
        mask[p - 1:p + c - 1] = False
        assert np.all(gH[r, mask] == 0.0)


def test_full_step_tiny_config():
    """Config "tiny" (fp32): policy and reference forward, loss, backward."""
    w = WL.make_config("tiny")
    dw = DeviceWorkload(w)
    op = _oracle_fwd(w, w.W)
    orf = _oracle_fwd(w, w.W_ref)
    ol = O.dpo_loss(op["seq_logp"], orf["seq_logp"], w.beta, w.layout)
    pol, _, lse = dw.forward(dw.W, want_grad=True)
    ref, _, _ = dw.forward(dw.W_ref, want_grad=False)
    out = dw.loss(pol, ref)
    assert abs(float(out["loss"].item()) - ol["loss"]) <= TOL_LOSS
    np.testing.assert_allclose(np64(out["margins"]), ol["margins"], atol=1e-4)
    dH, dW = dw.backward(lse, out["row_coef"])
    assert libdpo.check() == libdpo.OK
    oH, oW = O.backward(WL.widen(w.H, "f32"), WL.widen(w.W, "f32"), w.tokens, w.prompt_len,
                        w.completion_len, ol["row_coef"])
    assert rel_frob(np64(dH), oH) <= TOL_GRAD
    assert rel_frob(np64(dW), oW) <= TOL_GRAD


@pytest.mark.parametrize("layout", ["halves", "adjacent"])
def test_loss_kernel_on_identical_sums(layout):
    import torch
    rng = np.random.default_rng(3)
    for B in (1, 5, 64, 300):
        pol = (-rng.uniform(10, 3000, 2 * B)).astype(np.float32)
        ref = (pol + rng.normal(0, 30, 2 * B)).astype(np.float32)
        o = O.dpo_loss(pol.astype(np.float64), ref.astype(np.float64), 0.1, layout, grad_scale=0.5)
        out = {k: torch.full((n,), float("nan"), device="cuda") for k, n in
               [("loss", 1), ("accuracy", 1), ("margins", B), ("cr", B), ("rr", B), ("w", B),
                ("coef", 2 * B)]}
        libdpo.loss(B, layout, torch.from_numpy(pol).cuda(), torch.from_numpy(ref).cuda(), 0.1, 0.5,
                    out["loss"], out["accuracy"], out["margins"], out["cr"], out["rr"], out["w"],
                    out["coef"])
        assert abs(out["loss"].item() - o["loss"]) <= TOL_LOSS
        assert out["accuracy"].item() == pytest.approx(o["accuracy"], abs=1e-7)
        np.testing.assert_allclose(np64(out["margins"]), o["margins"], rtol=1e-6, atol=1e-6)
        np.testing.assert_allclose(np64(out["w"]), o["weights"], rtol=1e-6, atol=1e-7)
        np.testing.assert_allclose(np64(out["coef"]), o["row_coef"], rtol=1e-6, atol=1e-12)
        np.testing.assert_allclose(np64(out["cr"]), o["chosen_rewards"], rtol=1e-6, atol=1e-6)
        np.testing.assert_allclose(np64(out["rr"]), o["rejected_rewards"], rtol=1e-6, atol=1e-6)


def test_loss_worked_example_on_gpu():
    import torch
    pol = torch.tensor([-42.0, -47.5], device="cuda")
    ref = torch.tensor([-43.0, -46.0], device="cuda")
    out = {k: torch.zeros(1, device="cuda") for k in ("loss", "acc", "m", "cr", "rr", "w")}
    libdpo.loss(1, "halves", pol, ref, 0.1, 1.0, out["loss"], out["acc"], out["m"], out["cr"],
                out["rr"], out["w"])
    assert round(out["loss"].item(), 3) == 0.576
    assert round(out["w"].item(), 3) == 0.438
    assert round(out["m"].item(), 2) == 0.25
    assert out["acc"].item() == 1.0


def test_policy_equals_reference_gives_ln2():
    w = WL.make_custom(R=8, L=128, d=128, V=600, dtype="bf16", seed=9, prompt_range=(1, 60))
    dw = DeviceWorkload(w)
    pol, _, _ = dw.forward(dw.W, want_grad=False)
    ref, _, _ = dw.forward(dw.W, want_grad=False)
    out = dw.loss(pol, ref)
    assert out["loss"].item() == pytest.approx(math.log(2.0), abs=1e-7)
    assert np.all(np64(out["weights"]) == 0.5)
    assert out["accuracy"].item() == 0.0


def test_forward_is_deterministic():
    w = WL.make_custom(R=6, L=300, d=256, V=1000, dtype="bf16", seed=12, prompt_range=(1, 100))
    dw = DeviceWorkload(w)
    a = dw.forward(dw.W, want_grad=True)
    b = dw.forward(dw.W, want_grad=True)
    for x, y in zip(a, b):
        assert np.array_equal(np64(x), np64(y))


def test_empty_completions():
    import torch
    w = WL.make_custom(R=4, L=50, d=64, V=300, dtype="bf16", seed=13)
    w.completion_len[:] = 0
    dw = DeviceWorkload(w)
    seq, tok, lse = dw.forward(dw.W, want_grad=True)
    assert np.all(np64(seq) == 0.0) and np.all(np64(tok) == 0.0)
    dH, dW = dw.backward(lse, torch.ones(4, device="cuda"))
    assert np.all(np64(dH) == 0.0) and np.all(np64(dW) == 0.0)


def test_bad_target_is_reported_and_scored_zero():
    import torch
    w = WL.make_custom(R=2, L=40, d=64, V=300, dtype="bf16", seed=14, prompt_range=(2, 10),
                       min_completion=5)
    p = int(w.prompt_len[0])
    w.tokens[0, p + 1] = 300          # out of range, scored by position p
    dw = DeviceWorkload(w)
    libdpo.check()                     # clear
    seq, tok, _ = dw.forward(dw.W, want_grad=False)
    assert libdpo.check() == libdpo.ERR_BAD_TARGET
    assert np64(tok)[0, p] == 0.0
    assert libdpo.check() == libdpo.OK  # cleared by the read


def test_chunked_backward_matches_single_chunk():
    import torch
    w = WL.make_custom(R=4, L=400, d=128, V=700, dtype="bf16", seed=15, prompt_range=(1, 50),
                       full_rows=4)
    dw = DeviceWorkload(w)
    _, _, lse = dw.forward(dw.W, want_grad=True)
    coef = torch.linspace(-0.2, 0.3, 4, device="cuda")
    dH1, dW1 = dw.backward(lse, coef)
    b = dw.batch()
    _, full, mn = libdpo.workspace_size(b)
    small = mn + 2 * 128 * 2 * ((w.V + 7) // 8 * 8)      # room for 3 chunks of 128
    assert small < full
    dH2, dW2 = dw.backward(lse, coef, ws_bytes=small)
    assert rel_frob(np64(dH2), np64(dH1)) < 1e-6
    assert rel_frob(np64(dW2), np64(dW1)) < 1e-5


def test_accumulate_dW():
    import torch
    w = WL.make_custom(R=4, L=100, d=64, V=300, dtype="bf16", seed=16, prompt_range=(1, 40))
    dw = DeviceWorkload(w)
    _, _, lse = dw.forward(dw.W, want_grad=True)
    coef = torch.full((4,), 0.1, device="cuda")
    _, dW1 = dw.backward(lse, coef)
    base = torch.full_like(dW1, 0.25)
    _, dW2 = dw.backward(lse, coef, accumulate=True, dW=base.clone())
    # the accumulating store adds in fp32 with round-to-nearest-even: the same bits as
    # adding the freshly written dW to the old values
    assert torch.equal(dW2, dW1 + base)


def test_host_errors_leave_outputs_untouched():
    import torch
    w = WL.make_custom(R=2, L=30, d=64, V=100, dtype="bf16", seed=17)
    dw = DeviceWorkload(w)
    seq = torch.full((2,), 7.0, device="cuda")
    bad = w.prompt_len.copy()
    bad[0] = 0
    b = libdpo.BatchArgs(dw.H, dw.W, dw.tokens, bad, w.completion_len, dtype="bf16")
    ws = dw.workspace(1 << 20)
    with pytest.raises(libdpo.DpoError) as e:
        libdpo.seq_logprobs(b, False, seq, None, None, ws)
    assert e.value.status == libdpo.ERR_INVALID_ARG
    assert np.all(np64(seq) == 7.0)
