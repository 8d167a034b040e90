"""Pins for the CPU float64 oracle, against facts that do not come from the oracle.

Each test names what fixes the expected value: a number printed on the pages, a
closed form, a 50-digit brute force, a finite difference, or an invariant of the
mathematics. A plausible slip in the oracle (a dropped term, a sign, an
off-by-one in the next-token shift, a transposed operand) fails at least one.
"""
import json
import math
import os

import numpy as np
import pytest

from oracle import dpo_oracle as O
from preference_alignment_b200 import workloads as WL

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------- loss: pages' numbers
@pytest.mark.parametrize("layout", ["halves", "adjacent"])
def test_worked_example(layout):
    g = _golden("worked_example.json")
    pol = [g["policy"]["chosen"], g["policy"]["rejected"]]
    ref = [g["reference"]["chosen"], g["reference"]["rejected"]]
    # one pair: both layouts put chosen at row 0 and rejected at row 1
    out = O.dpo_loss(pol, ref, g["beta"], layout=layout)
    e, dec = g["expected"], g["printed_decimals"]
    assert round(out["chosen_rewards"][0], dec["chosen_reward"]) == e["chosen_reward"]
    assert round(out["rejected_rewards"][0], dec["rejected_reward"]) == e["rejected_reward"]
    assert round(out["margins"][0], dec["margin"]) == e["margin"]
    assert round(out["loss"], dec["loss"]) == e["loss"]
    assert round(out["weights"][0], dec["weight"]) == e["weight"]
    assert out["accuracy"] == 1.0
    # the rewards and margin are exact decimal arithmetic on the printed inputs
    assert abs(out["margins"][0] - 0.25) < 1e-12
    assert abs(out["chosen_rewards"][0] - 0.10) < 1e-12
    assert abs(out["rejected_rewards"][0] + 0.15) < 1e-12


def test_start_of_training_is_ln2():
    g = _golden("start_of_training.json")
    rng = np.random.default_rng(5)
    for B in (1, 3, 64):
        s = -rng.uniform(10, 2000, size=2 * B)
        for layout in ("halves", "adjacent"):
            out = O.dpo_loss(s, s.copy(), 0.1, layout=layout, grad_scale=0.25)
            assert out["loss"] == math.log(2.0)
            assert round(out["loss"], g["printed_decimals"]["loss"]) == g["expected"]["loss"]
            assert np.all(out["margins"] == 0.0)
            assert np.all(out["weights"] == 0.5)
            assert out["accuracy"] == 0.0          # strict margin > 0
            rows = O.pair_rows(B, layout)
            for c, r in rows:
                assert out["row_coef"][c] == pytest.approx(-0.25 * 0.1 * 0.5 / B, abs=0, rel=1e-15)
                assert out["row_coef"][r] == pytest.approx(+0.25 * 0.1 * 0.5 / B, abs=0, rel=1e-15)


def test_pair_swap_identity():
    # exchanging chosen and rejected negates the margin; softplus(m) = softplus(-m) + m
    rng = np.random.default_rng(7)
    B = 16
    pol = -rng.uniform(50, 500, 2 * B)
    ref = pol + rng.normal(0, 20, 2 * B)
    a = O.dpo_loss(pol, ref, 0.1, "halves")
    sw = np.concatenate([pol[B:], pol[:B]])
    sr = np.concatenate([ref[B:], ref[:B]])
    b = O.dpo_loss(sw, sr, 0.1, "halves")
    np.testing.assert_allclose(b["margins"], -a["margins"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(b["losses"], a["losses"] + a["margins"], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(a["weights"] + b["weights"], 1.0, rtol=0, atol=1e-15)


def test_layouts_are_row_permutations():
    rng = np.random.default_rng(8)
    B = 5
    pol = -rng.uniform(50, 500, 2 * B)
    ref = pol + rng.normal(0, 3, 2 * B)
    h = O.dpo_loss(pol, ref, 0.1, "halves")
    perm = np.empty(2 * B, dtype=int)
    perm[0::2] = np.arange(B)
    perm[1::2] = np.arange(B, 2 * B)
    a = O.dpo_loss(pol[perm], ref[perm], 0.1, "adjacent")
    assert a["loss"] == h["loss"]
    np.testing.assert_array_equal(a["margins"], h["margins"])
    np.testing.assert_array_equal(a["row_coef"], h["row_coef"][perm])


def test_loss_row_coef_by_finite_differences():
    rng = np.random.default_rng(9)
    B = 4
    pol = -rng.uniform(50, 100, 2 * B)
    ref = pol + rng.normal(0, 10, 2 * B)
    for layout in ("halves", "adjacent"):
        g = 0.5
        out = O.dpo_loss(pol, ref, 0.1, layout, grad_scale=g)
        eps = 1e-5
        for r in range(2 * B):
            p1, p2 = pol.copy(), pol.copy()
            p1[r] += eps
            p2[r] -= eps
            fd = g * (O.dpo_loss(p1, ref, 0.1, layout)["loss"] - O.dpo_loss(p2, ref, 0.1, layout)["loss"]) / (2 * eps)
            assert out["row_coef"][r] == pytest.approx(fd, rel=1e-6, abs=1e-12)


def test_softplus_sigmoid_extremes():
    # the stable forms stay finite far out: -log sigmoid(m) -> -m for m << 0, -> e^-m for m >> 0
    assert O.softplus(800.0) == 800.0
    assert O.softplus(-800.0) == 0.0
    assert O.sigmoid(-800.0) == 0.0 and O.sigmoid(800.0) == 1.0
    out = O.dpo_loss([-1000.0, 0.0], [0.0, 0.0], 1.0)   # margin -1000
    assert out["loss"] == 1000.0 and out["weights"][0] == 1.0


# ---------------------------------------------------------------- log-probs: closed forms
def _dense(H, W):
    return np.asarray(H, np.float64), np.asarray(W, np.float64)


def test_zero_weights_give_uniform_logprob():
    # W = 0: every logit is 0, so log p = -log V at every scored position
    w = WL.make_custom(R=6, L=40, d=16, V=37, dtype="f32", seed=3)
    H, W = _dense(w.H, w.W)
    W[:] = 0.0
    out = O.seq_logprobs(H, W, w.tokens, w.prompt_len, w.completion_len)
    for r in range(w.R):
        p, c = w.prompt_len[r], w.completion_len[r]
        np.testing.assert_allclose(out["tok_logp"][r, p - 1:p + c - 1], -math.log(37), rtol=0, atol=1e-15)
        assert out["seq_logp"][r] == pytest.approx(-c * math.log(37), rel=1e-14, abs=1e-14)
        mask = np.ones(w.L, bool)
        mask[p - 1:p + c - 1] = False
        assert np.all(out["tok_logp"][r, mask] == 0.0)


def test_single_token_vocab_gives_zero():
    w = WL.make_custom(R=2, L=12, d=4, V=1, dtype="f32", seed=4)
    out = O.seq_logprobs(*_dense(w.H, w.W), w.tokens, w.prompt_len, w.completion_len)
    assert np.all(out["tok_logp"] == 0.0) and np.all(out["seq_logp"] == 0.0)


def test_next_token_shift_closed_form():
    # V = 2, d = 1, W = [[1], [0]]: z_t = (a_t, 0), so log p(0) = log sigmoid(a_t) and
    # log p(1) = log sigmoid(-a_t). Every position gets a distinct a_t, so scoring the
    # wrong position (or the wrong token) changes the answer.
    R, L = 2, 9
    a = np.array([[0.5 + 0.25 * t for t in range(L)], [-1.0 - 0.5 * t for t in range(L)]])
    H = a[:, :, None]
    W = np.array([[1.0], [0.0]])
    tokens = np.array([[1, 0, 1, 1, 0, 0, 1, 0, 1], [0, 1, 1, 0, 1, 0, 0, 1, 1]])
    P = np.array([3, 1])
    C = np.array([4, 8])
    out = O.seq_logprobs(H, W, tokens, P, C)

    def logsig(x):
        return -math.log1p(math.exp(-x)) if x >= 0 else x - math.log1p(math.exp(x))

    for r in range(R):
        expect = np.zeros(L)
        for j in range(P[r], P[r] + C[r]):          # completion token j ...
            t = j - 1                               # ... is predicted by position j - 1
            y = tokens[r, j]
            expect[t] = logsig(a[r, t]) if y == 0 else logsig(-a[r, t])
        np.testing.assert_allclose(out["tok_logp"][r], expect, rtol=1e-14, atol=1e-15)
        assert out["seq_logp"][r] == pytest.approx(math.fsum(expect), rel=1e-14)


def test_rejects_rows_that_do_not_fit():
    with pytest.raises(ValueError):
        O.scored_positions([0], [3], 10)
    with pytest.raises(ValueError):
        O.scored_positions([4], [7], 10)
    assert O.scored_positions([4], [6], 10) == [(0, t) for t in range(3, 9)]
    assert O.scored_positions([4], [0], 10) == []


# ---------------------------------------------------------------- brute force
@pytest.mark.parametrize("seed", range(6))
def test_bruteforce_50_digits(seed):
    rng = np.random.default_rng(100 + seed)
    V = int(rng.integers(1, 9))
    d = int(rng.integers(1, 5))
    h = rng.normal(0, 2, size=(3, d))
    W = rng.normal(0, 2, size=(V, d))
    y = rng.integers(0, V, size=3)
    lp, _ = O.position_logprobs(h, W, y)
    for i in range(3):
        bf = float(O.logprob_bruteforce(h[i], W, y[i]))
        assert lp[i] == pytest.approx(bf, rel=1e-13, abs=1e-13)


def test_bruteforce_through_row_sums():
    w = WL.make_custom(R=4, L=10, d=3, V=6, dtype="f32", seed=11)
    H, W = _dense(w.H, w.W)
    out = O.seq_logprobs(H, W, w.tokens, w.prompt_len, w.completion_len)
    for r in range(w.R):
        p, c = w.prompt_len[r], w.completion_len[r]
        terms = [O.logprob_bruteforce(H[r, j - 1], W, w.tokens[r, j]) for j in range(p, p + c)]
        assert out["seq_logp"][r] == pytest.approx(float(sum(terms)), rel=1e-13, abs=1e-13)


# ---------------------------------------------------------------- invariants of log-softmax
def test_shift_invariance():
    # append a column of ones to H and a constant to every row of W: every logit of a
    # position moves by the same amount, so the log-softmax does not change
    w = WL.make_custom(R=4, L=30, d=8, V=50, dtype="f32", seed=12)
    H, W = _dense(w.H, w.W)
    base = O.seq_logprobs(H, W, w.tokens, w.prompt_len, w.completion_len)
    H2 = np.concatenate([H, np.ones(H.shape[:2] + (1,))], axis=2)
    W2 = np.concatenate([W, np.full((W.shape[0], 1), 3.7)], axis=1)
    sh = O.seq_logprobs(H2, W2, w.tokens, w.prompt_len, w.completion_len)
    np.testing.assert_allclose(sh["tok_logp"], base["tok_logp"], rtol=1e-12, atol=1e-12)


def test_vocab_permutation_invariance():
    w = WL.make_custom(R=4, L=30, d=8, V=50, dtype="f32", seed=13)
    H, W = _dense(w.H, w.W)
    base = O.seq_logprobs(H, W, w.tokens, w.prompt_len, w.completion_len)
    perm = np.random.default_rng(0).permutation(50)      # new row i holds old row perm[i]
    inv = np.argsort(perm)
    out = O.seq_logprobs(H, W[perm], inv[w.tokens], w.prompt_len, w.completion_len)
    np.testing.assert_allclose(out["tok_logp"], base["tok_logp"], rtol=1e-12, atol=1e-13)


def test_normalisation_over_vocab():
    rng = np.random.default_rng(14)
    V, d = 97, 12
    h = rng.normal(size=(1, d))
    W = rng.normal(size=(V, d))
    lp, _ = O.position_logprobs(np.repeat(h, V, 0), W, np.arange(V))
    assert np.all(lp <= 0)
    assert math.fsum(np.exp(lp)) == pytest.approx(1.0, abs=1e-14)


# ---------------------------------------------------------------- backward
def _tiny_problem(seed=21, dtype="f32"):
    w = WL.make_custom(R=4, L=12, d=5, V=9, dtype=dtype, seed=seed, layout="adjacent",
                       prompt_range=(1, 6), min_completion=1)
    H, W = _dense(w.H, w.W)
    Wr = np.asarray(w.W_ref, np.float64) + 0.3   # makes margins clearly non-zero
    return w, H, W, Wr


def _loss_of(w, H, W, ref, g):
    s = O.seq_logprobs(H, W, w.tokens, w.prompt_len, w.completion_len)["seq_logp"]
    return g * O.dpo_loss(s, ref, 0.5, w.layout)["loss"]


def test_backward_finite_differences():
    w, H, W, Wr = _tiny_problem()
    ref = O.seq_logprobs(H, Wr, w.tokens, w.prompt_len, w.completion_len)["seq_logp"]
    pol = O.seq_logprobs(H, W, w.tokens, w.prompt_len, w.completion_len)["seq_logp"]
    g = 0.75
    coef = O.dpo_loss(pol, ref, 0.5, w.layout, grad_scale=g)["row_coef"]
    dH, dW = O.backward(H, W, w.tokens, w.prompt_len, w.completion_len, coef)
    eps = 1e-6
    rng = np.random.default_rng(0)
    for _ in range(25):
        r, t, k = rng.integers(w.R), rng.integers(w.L), rng.integers(w.d)
        Hp, Hm = H.copy(), H.copy()
        Hp[r, t, k] += eps
        Hm[r, t, k] -= eps
        fd = (_loss_of(w, Hp, W, ref, g) - _loss_of(w, Hm, W, ref, g)) / (2 * eps)
        assert dH[r, t, k] == pytest.approx(fd, rel=1e-6, abs=1e-10)
    for _ in range(25):
        v, k = rng.integers(w.V), rng.integers(w.d)
        Wp, Wm = W.copy(), W.copy()
        Wp[v, k] += eps
        Wm[v, k] -= eps
        fd = (_loss_of(w, H, Wp, ref, g) - _loss_of(w, H, Wm, ref, g)) / (2 * eps)
        assert dW[v, k] == pytest.approx(fd, rel=1e-6, abs=1e-10)


def test_backward_invariants():
    w = WL.make_custom(R=6, L=40, d=7, V=31, dtype="f32", seed=22, prompt_range=(1, 20))
    H, W = _dense(w.H, w.W)
    coef = np.random.default_rng(1).normal(size=w.R)
    dH, dW = O.backward(H, W, w.tokens, w.prompt_len, w.completion_len, coef)
    # (i) every row of dz sums to zero over the vocabulary, so each column of dW sums to zero
    np.testing.assert_allclose(dW.sum(axis=0), 0.0, atol=1e-12)
    # (ii) a constant added to every row of W moves all logits of a position equally
    dH2, _ = O.backward(H, W + np.linspace(-1, 1, w.d)[None, :], w.tokens, w.prompt_len,
                        w.completion_len, coef)
    np.testing.assert_allclose(dH2, dH, rtol=1e-10, atol=1e-12)
    # (iii) bilinearity of z = h . w: <dW, W> = <dH, H> = sum dz * z
    assert float((dW * W).sum()) == pytest.approx(float((dH * H).sum()), rel=1e-11, abs=1e-11)
    # (iv) unscored positions get no gradient
    for r in range(w.R):
        p, c = w.prompt_len[r], w.completion_len[r]
        mask = np.ones(w.L, bool)
        mask[p - 1:p + c - 1] = False
        assert np.all(dH[r, mask] == 0.0)


def test_position_grad_h_matches_backward():
    w = WL.make_custom(R=3, L=20, d=6, V=25, dtype="f32", seed=23)
    H, W = _dense(w.H, w.W)
    coef = np.array([0.3, -0.2, 0.7])
    dH, _ = O.backward(H, W, w.tokens, w.prompt_len, w.completion_len, coef)
    for r, t in O.scored_positions(w.prompt_len, w.completion_len, w.L)[::3]:
        g = O.position_grad_h(H[r, t], W, w.tokens[r, t + 1], coef[r])
        np.testing.assert_allclose(g, dH[r, t], rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------- loss variants
def test_normalised_loss_with_unit_lengths_is_the_plain_loss():
    rng = np.random.default_rng(31)
    pol = -rng.uniform(1, 50, 8)
    ref = pol + rng.normal(0, 2, 8)
    a = O.dpo_loss(pol, ref, 0.1, "halves")
    b = O.dpo_loss(pol, ref, 0.1, "halves", completion_len=np.ones(8, int), normalize=True)
    assert a["loss"] == b["loss"]
    np.testing.assert_array_equal(a["row_coef"], b["row_coef"])


def test_normalised_loss_ignores_repeating_every_token():
    # doubling every completion (C -> 2C, S -> 2S) leaves average log-probs, hence the loss,
    # unchanged, while the plain sum-based loss changes
    rng = np.random.default_rng(32)
    C = rng.integers(1, 40, 8)
    pol = -rng.uniform(0.5, 3, 8) * C
    ref = pol + rng.normal(0, 1, 8)
    a = O.dpo_loss(pol, ref, 0.2, "adjacent", completion_len=C, normalize=True)
    b = O.dpo_loss(2 * pol, 2 * ref, 0.2, "adjacent", completion_len=2 * C, normalize=True)
    assert b["loss"] == pytest.approx(a["loss"], rel=1e-14)
    assert O.dpo_loss(2 * pol, 2 * ref, 0.2, "adjacent")["loss"] != pytest.approx(
        O.dpo_loss(pol, ref, 0.2, "adjacent")["loss"], rel=1e-6)


def test_nll_term_is_a_token_mean_over_chosen_completions():
    # pair 0: chosen C = 1, S = -1; pair 1: chosen C = 3, S = -9. Token mean: 10 / 4 = 2.5
    # (a per-pair mean of means would give 2.0). Policy == reference, so DPO gives ln 2.
    pol = np.array([-1.0, -9.0, -5.0, -7.0])           # halves: chosen rows 0, 1
    C = np.array([1, 3, 2, 2])
    out = O.dpo_loss(pol, pol.copy(), 0.1, "halves", completion_len=C, nll_weight=0.5)
    assert out["nll"] == 2.5
    assert out["loss"] == pytest.approx(math.log(2) + 0.5 * 2.5, rel=1e-15)


def test_nll_at_uniform_logits_is_log_vocab():
    # W = 0: every chosen token has log p = -log V, so the NLL is log V whatever the lengths
    w = WL.make_custom(R=6, L=40, d=8, V=53, dtype="f32", seed=33, prompt_range=(1, 20),
                       min_completion=1)
    H, W = _dense(w.H, w.W)
    W[:] = 0.0
    s = O.seq_logprobs(H, W, w.tokens, w.prompt_len, w.completion_len)["seq_logp"]
    out = O.dpo_loss(s, s.copy(), 0.1, "halves", completion_len=w.completion_len, nll_weight=1.0)
    assert out["nll"] == pytest.approx(math.log(53), rel=1e-13)


@pytest.mark.parametrize("normalize,nll", [(True, 0.0), (False, 0.7), (True, 0.3)])
def test_variant_row_coef_by_finite_differences(normalize, nll):
    rng = np.random.default_rng(34)
    B = 3
    C = rng.integers(1, 30, 2 * B)
    pol = -rng.uniform(0.5, 4, 2 * B) * C
    ref = pol + rng.normal(0, 3, 2 * B)
    for layout in ("halves", "adjacent"):
        kw = dict(completion_len=C, normalize=normalize, nll_weight=nll)
        out = O.dpo_loss(pol, ref, 0.1, layout, grad_scale=0.5, **kw)
        eps = 1e-5
        for r in range(2 * B):
            p1, p2 = pol.copy(), pol.copy()
            p1[r] += eps
            p2[r] -= eps
            fd = 0.5 * (O.dpo_loss(p1, ref, 0.1, layout, **kw)["loss"]
                        - O.dpo_loss(p2, ref, 0.1, layout, **kw)["loss"]) / (2 * eps)
            assert out["row_coef"][r] == pytest.approx(fd, rel=1e-6, abs=1e-12)


@pytest.mark.parametrize("normalize", [False, True])
def test_reference_free_is_any_reference_that_ties_each_pair(normalize):
    """The reference-free objective equals the referenced one whenever each pair's two
    reference values (as the loss uses them) are equal, whatever that value: the
    margins, losses, weights, accuracy and row coefficients agree, and the rewards
    differ by beta times the tied value."""
    rng = np.random.default_rng(36)
    B = 6
    C = rng.integers(1, 40, 2 * B)
    pol = -rng.uniform(0.5, 4, 2 * B) * C
    tie = rng.normal(0, 50, B)
    for layout in ("halves", "adjacent"):
        ref = np.empty(2 * B)
        for i, (c, r) in enumerate(O.pair_rows(B, layout)):
            # the value the loss sees is ref / C when normalising, ref otherwise
            ref[c] = tie[i] * (C[c] if normalize else 1)
            ref[r] = tie[i] * (C[r] if normalize else 1)
        kw = dict(completion_len=C, normalize=normalize, nll_weight=0.3)
        free = O.dpo_loss(pol, None, 0.1, layout, grad_scale=0.5, **kw)
        tied = O.dpo_loss(pol, ref, 0.1, layout, grad_scale=0.5, **kw)
        for k in ("margins", "losses", "weights", "row_coef"):
            np.testing.assert_allclose(free[k], tied[k], rtol=1e-12, atol=1e-14)
        for k in ("loss", "accuracy", "nll"):
            assert free[k] == pytest.approx(tied[k], rel=1e-12, abs=1e-15)
        np.testing.assert_allclose(free["chosen_rewards"], tied["chosen_rewards"] + 0.1 * tie,
                                   rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(free["rejected_rewards"],
                                   tied["rejected_rewards"] + 0.1 * tie, rtol=1e-12, atol=1e-12)


def test_reference_free_on_the_worked_example_policy():
    """The worked example's policy sums (-42.0 chosen, -47.5 rejected, beta 0.1) with no
    reference: rewards are beta times the sums, the margin 0.55, one correct pair."""
    out = O.dpo_loss([-42.0, -47.5], None, 0.1, "adjacent")
    assert out["chosen_rewards"][0] == pytest.approx(-4.2, abs=1e-15)
    assert out["rejected_rewards"][0] == pytest.approx(-4.75, abs=1e-15)
    assert out["margins"][0] == pytest.approx(0.55, abs=1e-15)
    assert out["accuracy"] == 1.0
    # the referenced example's loss (0.576, margin 0.25) is larger: the margin grew
    assert out["loss"] < O.dpo_loss([-42.0, -47.5], [-43.0, -46.0], 0.1, "adjacent")["loss"]


@pytest.mark.parametrize("normalize,nll", [(False, 0.0), (True, 0.5)])
def test_reference_free_row_coef_by_finite_differences(normalize, nll):
    rng = np.random.default_rng(37)
    B = 3
    C = rng.integers(1, 30, 2 * B)
    pol = -rng.uniform(0.05, 0.4, 2 * B) * C
    kw = dict(completion_len=C, normalize=normalize, nll_weight=nll)
    for layout in ("halves", "adjacent"):
        out = O.dpo_loss(pol, None, 0.1, layout, grad_scale=0.5, **kw)
        eps = 1e-5
        for r in range(2 * B):
            p1, p2 = pol.copy(), pol.copy()
            p1[r] += eps
            p2[r] -= eps
            fd = 0.5 * (O.dpo_loss(p1, None, 0.1, layout, **kw)["loss"]
                        - O.dpo_loss(p2, None, 0.1, layout, **kw)["loss"]) / (2 * eps)
            assert out["row_coef"][r] == pytest.approx(fd, rel=1e-6, abs=1e-12)


@pytest.mark.parametrize("normalize,nll", [(False, 0.0), (True, 0.0), (False, 0.6), (True, 0.4)])
def test_data_parallel_shares_add_up_to_the_whole_batch(normalize, nll):
    """Shares of a partition of the pairs into unequal parts (1, 2 and 4 pairs), each
    computed with the whole batch's pair and chosen-token counts, add up to the loss,
    accuracy and NLL of the whole batch; the row coefficients of each part are the
    whole batch's coefficients of its rows, and per-pair values are unchanged."""
    rng = np.random.default_rng(35)
    B = 7
    C = rng.integers(1, 30, 2 * B)
    pol = -rng.uniform(0.5, 4, 2 * B) * C
    ref = pol + rng.normal(0, 3, 2 * B)
    kw = dict(completion_len=C, normalize=normalize, nll_weight=nll)
    whole = O.dpo_loss(pol, ref, 0.1, "adjacent", grad_scale=0.5, **kw)
    Ng = int(sum(C[0::2]))
    tot = {"loss": 0.0, "accuracy": 0.0, "nll": 0.0}
    for pairs in ([0], [1, 2], [3, 4, 5, 6]):
        rows = np.array([r for i in pairs for r in (2 * i, 2 * i + 1)])
        part = O.dpo_loss(pol[rows], ref[rows], 0.1, "adjacent", grad_scale=0.5,
                          completion_len=C[rows], normalize=normalize, nll_weight=nll,
                          pairs_total=B, nll_tokens_total=Ng)
        for k in tot:
            tot[k] += part[k]
        np.testing.assert_allclose(part["row_coef"], whole["row_coef"][rows], rtol=1e-14,
                                   atol=1e-17)
        np.testing.assert_allclose(part["margins"], whole["margins"][pairs], rtol=1e-15)
        np.testing.assert_allclose(part["weights"], whole["weights"][pairs], rtol=1e-15)
    for k in tot:
        assert tot[k] == pytest.approx(whole[k], rel=1e-13, abs=1e-15)


# ---------------------------------------------------------------- logits-mean metrics
def test_logits_mean_equal_vocab_rows_closed_form():
    """Every vocabulary row equal to w makes every logit of position t equal h_t . w,
    so each side's mean is the mean of h_t . w over its rows and ALL positions."""
    rng = np.random.default_rng(40)
    R, L, d, V = 6, 9, 5, 11
    H = rng.normal(size=(R, L, d))
    w = rng.normal(size=d)
    W = np.tile(w, (V, 1))
    for layout, chosen in (("halves", [0, 1, 2]), ("adjacent", [0, 2, 4])):
        rejected = [r for r in range(R) if r not in chosen]
        want = []
        for rows in (chosen, rejected):
            vals = [sum(H[r, t, k] * w[k] for k in range(d)) for r in rows for t in range(L)]
            want.append(math.fsum(vals) / len(vals))
        got = O.logits_mean(H, W, layout)
        assert got[0] == pytest.approx(want[0], rel=1e-12, abs=1e-14)
        assert got[1] == pytest.approx(want[1], rel=1e-12, abs=1e-14)


def test_logits_mean_counts_prompt_and_pad_positions():
    """A single nonzero hidden state at the last (pad, never scored) position of one
    chosen row: the chosen mean is (h . sum_v W[v]) / (B L V), the rejected mean 0."""
    R, L, d, V = 4, 6, 3, 5
    H = np.zeros((R, L, d))
    H[1, L - 1] = [2.0, -1.0, 0.5]
    W = np.arange(V * d, dtype=np.float64).reshape(V, d) / 8.0 - 1.0
    colsum = [sum(W[v, k] for v in range(V)) for k in range(d)]
    want = sum(H[1, L - 1, k] * colsum[k] for k in range(d)) / (2 * L * V)
    c, r = O.logits_mean(H, W, "halves")       # row 1 is chosen under halves (B = 2)
    assert c == pytest.approx(want, rel=1e-14) and c != 0.0
    assert r == 0.0
    c, r = O.logits_mean(H, W, "adjacent")     # ... and rejected under adjacent pairs
    assert c == 0.0 and r == pytest.approx(want, rel=1e-14)


@pytest.mark.parametrize("seed", range(3))
def test_logits_mean_bruteforce_50_digits(seed):
    """Every logit summed in 50-digit decimal arithmetic, divided by the count."""
    import decimal
    rng = np.random.default_rng(50 + seed)
    R, L, d, V = 4, 3, 3, 4
    H = rng.normal(size=(R, L, d))
    W = rng.normal(size=(V, d))
    ctx = decimal.Context(prec=50)
    D = decimal.Decimal
    for layout, sides in (("halves", ([0, 1], [2, 3])), ("adjacent", ([0, 2], [1, 3]))):
        got = O.logits_mean(H, W, layout)
        for rows, g in zip(sides, got):
            tot = D(0)
            for r in rows:
                for t in range(L):
                    for v in range(V):
                        for k in range(d):
                            tot = ctx.add(tot, ctx.multiply(D(float(H[r, t, k])), D(float(W[v, k]))))
            want = float(ctx.divide(tot, D(len(rows) * L * V)))
            assert g == pytest.approx(want, rel=1e-13, abs=1e-15)


def test_logits_mean_is_bilinear():
    """sum_{t,v} h_t . W[v] = (sum_t h_t) . (sum_v W[v]): the mean follows from the
    two sums, and scaling H or W scales it."""
    rng = np.random.default_rng(41)
    R, L, d, V = 4, 300, 7, 13          # L > 256: more than one position chunk per row
    H = rng.normal(size=(R, L, d))
    W = rng.normal(size=(V, d))
    c, r = O.logits_mean(H, W)
    u_c, u_r = H[:2].reshape(-1, d).sum(0), H[2:].reshape(-1, d).sum(0)
    s = W.sum(0)
    assert c == pytest.approx(float(u_c @ s) / (2 * L * V), rel=1e-10)
    assert r == pytest.approx(float(u_r @ s) / (2 * L * V), rel=1e-10)
    c2, r2 = O.logits_mean(3.0 * H, -0.5 * W)
    assert c2 == pytest.approx(-1.5 * c, rel=1e-12) and r2 == pytest.approx(-1.5 * r, rel=1e-12)
