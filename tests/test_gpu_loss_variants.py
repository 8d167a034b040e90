"""dpo_loss_ex (length-normalised sums, SFT/NLL term on the chosen completions)
against the oracle: on identical sums, and end to end through the backward."""
import numpy as np
import pytest

from oracle import dpo_oracle as O
from preference_alignment_b200 import libdpo
from preference_alignment_b200 import workloads as WL

from dpo_harness import DeviceWorkload, TOL_GRAD, TOL_LOSS, np64, rel_frob

pytestmark = pytest.mark.gpu


def _run_ex(B, layout, pol, ref, C, beta, gscale, normalize, nll_weight, pairs_total=0,
            nll_tokens_total=0, reference_free=False):
    import torch
    dev = "cuda"
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(dev)  # noqa: E731
    out = {k: torch.full((n,), float("nan"), device=dev) for k, n in
           [("loss", 1), ("acc", 1), ("m", B), ("cr", B), ("rr", B), ("w", B), ("coef", 2 * B),
            ("nll", 1)]}
    clen = torch.from_numpy(np.asarray(C, np.int32)).to(dev)
    libdpo.loss_ex(B, layout, t(pol), None if ref is None else t(ref), beta, gscale, out["loss"],
                   out["acc"], out["m"], out["cr"], out["rr"], out["w"], out["coef"], out["nll"],
                   normalize=normalize, nll_weight=nll_weight, completion_len=clen,
                   pairs_total=pairs_total, nll_tokens_total=nll_tokens_total,
                   reference_free=reference_free)
    return {k: np64(v) for k, v in out.items()}


@pytest.mark.parametrize("layout", ["halves", "adjacent"])
@pytest.mark.parametrize("normalize,nll", [(False, 0.0), (True, 0.0), (False, 0.5), (True, 1.0)])
def test_variants_on_identical_sums(layout, normalize, nll):
    rng = np.random.default_rng(71)
    for B in (1, 7, 300):
        C = rng.integers(0, 600, 2 * B)
        C[0] = 5
        pol = (-rng.uniform(0.5, 4.0, 2 * B) * C).astype(np.float32)
        ref = (pol + rng.normal(0, 5, 2 * B)).astype(np.float32)
        o = O.dpo_loss(pol.astype(np.float64), ref.astype(np.float64), 0.1, layout, grad_scale=0.5,
                       completion_len=C, normalize=normalize, nll_weight=nll)
        g = _run_ex(B, layout, pol, ref, C, 0.1, 0.5, normalize, nll)
        assert abs(g["loss"][0] - o["loss"]) <= TOL_LOSS
        assert abs(g["nll"][0] - o["nll"]) <= 1e-5 * max(1.0, abs(o["nll"]))
        assert g["acc"][0] == pytest.approx(o["accuracy"], abs=1e-7)
        np.testing.assert_allclose(g["m"], o["margins"], rtol=1e-5, atol=1e-6)
        np.testing.assert_allclose(g["w"], o["weights"], rtol=1e-5, atol=1e-7)
        np.testing.assert_allclose(g["coef"], o["row_coef"], rtol=1e-5, atol=1e-10)


def test_variants_end_to_end_through_the_backward():
    import torch
    w = WL.make_custom(R=8, L=200, d=256, V=1200, dtype="bf16", seed=72, prompt_range=(1, 80),
                       min_completion=1, ref_std=0.05)
    dw = DeviceWorkload(w)
    H = WL.widen(w.H, "bf16")
    Wd = WL.widen(w.W, "bf16")
    op = O.seq_logprobs(H, Wd, w.tokens, w.prompt_len, w.completion_len)
    orf = O.seq_logprobs(H, WL.widen(w.W_ref, "bf16"), w.tokens, w.prompt_len, w.completion_len)
    ol = O.dpo_loss(op["seq_logp"], orf["seq_logp"], w.beta, w.layout, completion_len=w.completion_len,
                    normalize=True, nll_weight=0.5)
    pol, _, lse = dw.forward(dw.W, want_grad=True)
    ref, _, _ = dw.forward(dw.W_ref, want_grad=False)
    B = w.R // 2
    out = {k: torch.empty(n, device="cuda") for k, n in [("loss", 1), ("coef", 2 * B), ("nll", 1)]}
    clen = torch.from_numpy(w.completion_len).cuda()
    libdpo.loss_ex(B, w.layout, pol, ref, w.beta, 1.0, out["loss"], row_coef=out["coef"],
                   nll=out["nll"], normalize=True, nll_weight=0.5, completion_len=clen)
    assert abs(out["loss"].item() - ol["loss"]) <= TOL_LOSS
    dH, dW = dw.backward(lse, out["coef"])
    assert libdpo.check() == libdpo.OK
    oH, oW = O.backward(H, Wd, w.tokens, w.prompt_len, w.completion_len, ol["row_coef"])
    assert rel_frob(np64(dH), oH) <= TOL_GRAD
    assert rel_frob(np64(dW), oW) <= TOL_GRAD


@pytest.mark.parametrize("normalize,nll", [(False, 0.0), (False, 0.5), (True, 0.25)])
def test_data_parallel_shares_against_the_oracle(normalize, nll):
    """dpo_loss_ex with the whole batch's pair and chosen-token counts: each part of an
    unequal partition gives the oracle's share, and the shares add up to the oracle's
    single-process values of the whole batch."""
    rng = np.random.default_rng(73)
    B = 9
    C = rng.integers(1, 500, 2 * B)
    pol = (-rng.uniform(0.5, 4.0, 2 * B) * C).astype(np.float32)
    ref = (pol + rng.normal(0, 5, 2 * B)).astype(np.float32)
    Ng = int(C[0::2].sum())
    whole = O.dpo_loss(pol.astype(np.float64), ref.astype(np.float64), 0.1, "adjacent",
                       completion_len=C, normalize=normalize, nll_weight=nll)
    tot = np.zeros(3)
    for pairs in ([0, 1, 2, 3, 4, 5], [6], [7, 8]):
        rows = np.array([r for i in pairs for r in (2 * i, 2 * i + 1)])
        o = O.dpo_loss(pol[rows].astype(np.float64), ref[rows].astype(np.float64), 0.1,
                       "adjacent", completion_len=C[rows], normalize=normalize, nll_weight=nll,
                       pairs_total=B, nll_tokens_total=Ng)
        g = _run_ex(len(pairs), "adjacent", pol[rows], ref[rows], C[rows], 0.1, 1.0, normalize,
                    nll, pairs_total=B, nll_tokens_total=Ng)
        assert abs(g["loss"][0] - o["loss"]) <= TOL_LOSS
        assert g["acc"][0] == pytest.approx(o["accuracy"], abs=1e-7)
        np.testing.assert_allclose(g["coef"], o["row_coef"], rtol=1e-5, atol=1e-10)
        np.testing.assert_allclose(g["coef"], whole["row_coef"][rows], rtol=1e-5, atol=1e-10)
        tot += [g["loss"][0], g["acc"][0], g["nll"][0]]
    assert abs(tot[0] - whole["loss"]) <= TOL_LOSS
    assert tot[1] == pytest.approx(whole["accuracy"], abs=1e-6)
    assert abs(tot[2] - whole["nll"]) <= 1e-5 * max(1.0, abs(whole["nll"]))


@pytest.mark.parametrize("layout", ["halves", "adjacent"])
@pytest.mark.parametrize("normalize,nll", [(False, 0.0), (True, 0.0), (True, 0.5)])
def test_reference_free_on_identical_sums(layout, normalize, nll):
    """reference_free against the oracle's reference-free loss (ref=None); a reference
    buffer full of NaN passed beside the flag must not be read."""
    rng = np.random.default_rng(74)
    for B in (1, 5, 300):
        C = rng.integers(1, 600, 2 * B)
        pol = (-rng.uniform(0.01, 0.05, 2 * B) * C).astype(np.float32)
        o = O.dpo_loss(pol.astype(np.float64), None, 0.1, layout, grad_scale=0.5,
                       completion_len=C, normalize=normalize, nll_weight=nll)
        nan_ref = np.full(2 * B, np.nan, np.float32)
        for ref in (None, nan_ref):
            g = _run_ex(B, layout, pol, ref, C, 0.1, 0.5, normalize, nll, reference_free=True)
            assert abs(g["loss"][0] - o["loss"]) <= TOL_LOSS
            assert g["acc"][0] == pytest.approx(o["accuracy"], abs=1e-7)
            np.testing.assert_allclose(g["m"], o["margins"], rtol=1e-5, atol=1e-6)
            np.testing.assert_allclose(g["cr"], o["chosen_rewards"], rtol=1e-5, atol=1e-6)
            np.testing.assert_allclose(g["rr"], o["rejected_rewards"], rtol=1e-5, atol=1e-6)
            np.testing.assert_allclose(g["w"], o["weights"], rtol=1e-5, atol=1e-7)
            np.testing.assert_allclose(g["coef"], o["row_coef"], rtol=1e-5, atol=1e-10)


def test_reference_free_end_to_end_through_the_backward():
    """No reference forward at all: policy sums -> reference-free loss -> backward, against
    the oracle's pipeline on the same inputs."""
    import torch
    w = WL.make_custom(R=6, L=160, d=128, V=900, dtype="bf16", seed=75, prompt_range=(1, 60),
                       min_completion=1)
    dw = DeviceWorkload(w)
    H = WL.widen(w.H, "bf16")
    Wd = WL.widen(w.W, "bf16")
    op = O.seq_logprobs(H, Wd, w.tokens, w.prompt_len, w.completion_len)
    ol = O.dpo_loss(op["seq_logp"], None, w.beta, w.layout)
    pol, _, lse = dw.forward(dw.W, want_grad=True)
    B = w.R // 2
    out = {k: torch.empty(n, device="cuda") for k, n in [("loss", 1), ("coef", 2 * B)]}
    libdpo.loss_ex(B, w.layout, pol, None, w.beta, 1.0, out["loss"], row_coef=out["coef"],
                   reference_free=True)
    assert abs(out["loss"].item() - ol["loss"]) <= TOL_LOSS
    dH, dW = dw.backward(lse, out["coef"])
    assert libdpo.check() == libdpo.OK
    oH, oW = O.backward(H, Wd, w.tokens, w.prompt_len, w.completion_len, ol["row_coef"])
    assert rel_frob(np64(dH), oH) <= TOL_GRAD
    assert rel_frob(np64(dW), oW) <= TOL_GRAD
