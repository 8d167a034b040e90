"""Identities of the oracle's DPO loss over random inputs (hypothesis), each fixed by the
mathematics of the sigmoid loss rather than by the oracle itself: the pair-swap identity,
the data-parallel partition of the shares, the reference-free reading as a tied reference,
and the ranges of the outputs. Host only."""
import math

import numpy as np
import pytest
from hypothesis import given, settings
from hypothesis import strategies as st

from oracle import dpo_oracle as O

FINITE = dict(allow_nan=False, allow_infinity=False)


def _pairs(draw, B, lo=-5000.0, hi=0.0):
    vals = st.floats(lo, hi, **FINITE)
    pol = np.array(draw(st.lists(vals, min_size=2 * B, max_size=2 * B)))
    ref = np.array(draw(st.lists(vals, min_size=2 * B, max_size=2 * B)))
    return pol, ref


@st.composite
def batches(draw, max_pairs=12):
    B = draw(st.integers(1, max_pairs))
    pol, ref = _pairs(draw, B)
    beta = draw(st.floats(1e-3, 2.0, **FINITE))
    C = np.array(draw(st.lists(st.integers(0, 4096), min_size=2 * B, max_size=2 * B)))
    return B, pol, ref, beta, C


@settings(max_examples=200, deadline=None)
@given(batches(), st.sampled_from(["halves", "adjacent"]))
def test_swapping_chosen_and_rejected(batch, layout):
    """Exchanging each pair's rows negates its margin, and softplus(m) = softplus(-m) + m
    relates the two losses; the two weights of a pair add up to 1."""
    B, pol, ref, beta, _ = batch
    a = O.dpo_loss(pol, ref, beta, layout)
    swap = np.arange(2 * B)
    for c, r in O.pair_rows(B, layout):
        swap[c], swap[r] = r, c
    b = O.dpo_loss(pol[swap], ref[swap], beta, layout)
    scale = 1.0 + np.abs(a["margins"])
    np.testing.assert_allclose(b["margins"], -a["margins"], rtol=0, atol=1e-12 * scale.max())
    np.testing.assert_allclose(b["losses"], a["losses"] + a["margins"], rtol=1e-12,
                               atol=1e-12 * scale.max())
    np.testing.assert_allclose(a["weights"] + b["weights"], 1.0, rtol=0, atol=1e-15)


@settings(max_examples=200, deadline=None)
@given(batches(), st.sampled_from(["halves", "adjacent"]))
def test_output_ranges_and_accuracy_count(batch, layout):
    B, pol, ref, beta, _ = batch
    out = O.dpo_loss(pol, ref, beta, layout)
    assert out["loss"] >= 0.0
    assert np.all((out["weights"] >= 0.0) & (out["weights"] <= 1.0))
    assert np.all(out["losses"] >= 0.0)
    # -log sigmoid(m) >= max(-m, 0) and <= max(-m, 0) + log 2
    lower = np.maximum(-out["margins"], 0.0)
    assert np.all(out["losses"] >= lower - 1e-12 * (1 + lower))
    assert np.all(out["losses"] <= lower + math.log(2) + 1e-12 * (1 + lower))
    assert out["accuracy"] * B == sum(1 for m in out["margins"] if m > 0)


@settings(max_examples=150, deadline=None)
@given(batches(), st.booleans(), st.floats(0.0, 2.0, **FINITE), st.data())
def test_shares_of_any_partition_add_up(batch, normalize, nll, data):
    """Each part's loss, accuracy and NLL, computed with the whole batch's pair and chosen-
    token counts, sum to the whole batch's; each part's row coefficients are the whole
    batch's coefficients of its rows."""
    B, pol, ref, beta, C = batch
    owner = np.array(data.draw(st.lists(st.integers(0, 2), min_size=B, max_size=B)))
    kw = dict(completion_len=C, normalize=normalize, nll_weight=nll)
    whole = O.dpo_loss(pol, ref, beta, "adjacent", **kw)
    Ng = int(C[0::2].sum())
    tot = {"loss": 0.0, "accuracy": 0.0, "nll": 0.0}
    for q in range(3):
        pairs = np.flatnonzero(owner == q)
        if len(pairs) == 0:
            continue
        rows = np.array([r for i in pairs for r in (2 * i, 2 * i + 1)])
        part = O.dpo_loss(pol[rows], ref[rows], beta, "adjacent", completion_len=C[rows],
                          normalize=normalize, nll_weight=nll, pairs_total=B,
                          nll_tokens_total=Ng)
        for k in tot:
            tot[k] += part[k]
        np.testing.assert_allclose(part["row_coef"], whole["row_coef"][rows], rtol=1e-12,
                                   atol=1e-15)
    for k in tot:
        assert tot[k] == pytest.approx(whole[k], rel=1e-11, abs=1e-12)


@settings(max_examples=150, deadline=None)
@given(batches(), st.booleans(), st.sampled_from(["halves", "adjacent"]), st.data())
def test_reference_free_is_a_tied_reference(batch, normalize, layout, data):
    B, pol, _, beta, C = batch
    C = np.maximum(C, 1)
    tie = np.array(data.draw(st.lists(st.floats(-100.0, 100.0, **FINITE), min_size=B,
                                      max_size=B)))
    ref = np.empty(2 * B)
    for i, (c, r) in enumerate(O.pair_rows(B, layout)):
        ref[c] = tie[i] * (C[c] if normalize else 1)
        ref[r] = tie[i] * (C[r] if normalize else 1)
    kw = dict(completion_len=C, normalize=normalize)
    free = O.dpo_loss(pol, None, beta, layout, **kw)
    tied = O.dpo_loss(pol, ref, beta, layout, **kw)
    scale = 1.0 + np.abs(free["margins"]).max() + beta * np.abs(tie).max()
    np.testing.assert_allclose(free["margins"], tied["margins"], rtol=0, atol=1e-9 * scale)
    np.testing.assert_allclose(free["weights"], tied["weights"], rtol=0, atol=1e-9 * scale)
    assert abs(free["loss"] - tied["loss"]) <= 1e-9 * scale
