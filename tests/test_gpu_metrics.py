"""Logits-mean metrics (dpo_logits_mean) against the oracle, through the C ABI.

The oracle forms every logit of every position and averages them; the CUDA path
never forms a logit (it uses the bilinearity sum_{t,v} z_tv = (sum_t h_t).(sum_v W_v),
pinned on the oracle side). Tolerance, from the arithmetic: the CUDA side adds groups
of at most 8 rows in fp32 (error <= 7 * 2^-24 of the group's sum of absolute values;
exact for most groups, as bf16 has 8-bit mantissas) and everything else in fp64, then
rounds the mean to fp32 (2^-24 relative). To first order
    |gpu - oracle| <= 2^-23 |oracle| + 5e-7 * sum_k (A_k |s_k| + |u_k| S_k) / (B L V)
with u_k, A_k the side's column sum of H and of |H|, s_k, S_k those of W. In the
small cases below one dropped position moves the mean by ~100x that bound. At the
full Llama-3.1-8B head size the oracle forms all 2.1e9 logits of each side too (a
17 TFLOP fp64 product on the host, plus the exact sums).
"""
import numpy as np
import pytest

from oracle import dpo_oracle as O
from preference_alignment_b200 import libdpo
from preference_alignment_b200 import workloads as WL

from dpo_harness import DeviceWorkload

pytestmark = pytest.mark.gpu


def _side_rows(R, layout):
    B = R // 2
    if layout == "halves":
        return list(range(B)), list(range(B, R))
    return list(range(0, R, 2)), list(range(1, R, 2))


def _bound_terms(u, s, A, S):
    return float(np.abs(s) @ A + np.abs(u) @ S)


def _scale(H, W, layout):
    """sum_k (A_k |s_k| + |u_k| S_k) / (B L V) for each side (fp64, from the inputs)."""
    R, L, d = H.shape
    s, S = W.sum(axis=0), np.abs(W).sum(axis=0)
    out = []
    for rows in _side_rows(R, layout):
        h = H[rows].reshape(-1, d)
        out.append(_bound_terms(h.sum(axis=0), s, np.abs(h).sum(axis=0), S)
                   / (R // 2 * L * W.shape[0]))
    return out


def _run(w, layout):
    import torch
    dw = DeviceWorkload(w)
    b = dw.batch()
    fwd, _, _ = libdpo.workspace_size(b)
    ws = dw.workspace(fwd)
    means = torch.full((2,), float("nan"), device="cuda")
    libdpo.logits_mean(b, layout, means, ws)
    assert libdpo.check() == libdpo.OK
    return means.double().cpu().numpy(), dw, b, ws


def _assert_close(got, want, scale):
    for g, e, sc in zip(got, want, scale):
        assert abs(g - e) <= 2.0 ** -23 * abs(e) + 5e-7 * sc, (g, e, sc)


@pytest.mark.parametrize("R,L,d,V,dtype,layout,seed", [
    (4, 40, 256, 1000, "bf16", "halves", 1),
    (4, 40, 256, 1000, "bf16", "adjacent", 2),
    (6, 33, 200, 777, "bf16", "halves", 3),      # d not a multiple of the 256-column slab
    (2, 300, 520, 5001, "bf16", "adjacent", 4),  # one pair, several slabs, ragged last slab
    (8, 17, 8, 64, "bf16", "halves", 5),         # smallest hidden size
    (4, 32, 64, 1000, "f32", "adjacent", 6),
])
def test_logits_mean_matches_oracle(R, L, d, V, dtype, layout, seed):
    w = WL.make_custom(R=R, L=L, d=d, V=V, dtype=dtype, seed=seed, layout=layout,
                       prompt_range=(1, L // 3))
    H, W = WL.widen(w.H, dtype), WL.widen(w.W, dtype)
    got, _, _, _ = _run(w, layout)
    _assert_close(got, O.logits_mean(H, W, layout), _scale(H, W, layout))


def test_logits_mean_tiny_config():
    w = WL.make_config("tiny")
    H, W = WL.widen(w.H, w.dtype), WL.widen(w.W, w.dtype)
    got, _, _, _ = _run(w, w.layout)
    _assert_close(got, O.logits_mean(H, W, w.layout), _scale(H, W, w.layout))


def test_logits_mean_is_deterministic_and_ignores_the_completion_mask():
    import torch
    w = WL.make_custom(R=4, L=100, d=512, V=3000, dtype="bf16", seed=7, prompt_range=(1, 40))
    got, dw, b, ws = _run(w, "halves")
    again = torch.empty(2, device="cuda")
    libdpo.logits_mean(b, "halves", again, ws)
    assert np.array_equal(got, again.double().cpu().numpy())
    # every position counts: other prompt / completion lengths give the same result
    b2 = dw.batch(prompt_len=np.full(w.R, 1, np.int32), completion_len=np.zeros(w.R, np.int32))
    libdpo.logits_mean(b2, "halves", again, ws)
    assert libdpo.check() == libdpo.OK
    assert np.array_equal(got, again.double().cpu().numpy())


def test_logits_mean_llama8b_head_against_the_oracle():
    """Full size (8 x 2048 positions, d 4096, V 128,256) in the workspace bench.py uses,
    against oracle.logits_mean over every logit."""
    w = WL.make_config("llama8b", with_ref=False)
    got, _, _, _ = _run(w, "halves")
    H, W = WL.widen(w.H, "bf16"), WL.widen(w.W, "bf16")
    _assert_close(got, O.logits_mean(H, W, "halves"), _scale(H, W, "halves"))


def test_logits_mean_largest_hidden_size():
    """d = 65,536: 256 column slabs, one row split each."""
    w = WL.make_custom(R=2, L=8, d=65536, V=64, dtype="bf16", seed=8, prompt_range=(1, 1),
                       min_completion=1)
    H, W = WL.widen(w.H, "bf16"), WL.widen(w.W, "bf16")
    got, _, _, _ = _run(w, "halves")
    _assert_close(got, O.logits_mean(H, W, "halves"), _scale(H, W, "halves"))


def test_logits_mean_largest_vocabulary():
    """V = 2^24 rows of W in one column slab: the bilinear form, block by block."""
    w = WL.make_custom(R=2, L=8, d=8, V=1 << 24, dtype="bf16", seed=9, prompt_range=(1, 1),
                       min_completion=1)
    got, _, _, _ = _run(w, "adjacent")
    s, S = np.zeros(w.d), np.zeros(w.d)
    for v0 in range(0, w.V, 1 << 20):
        blk = WL.widen(w.W[v0:v0 + (1 << 20)], "bf16")
        s += blk.sum(axis=0)
        S += np.abs(blk).sum(axis=0)
    H = WL.widen(w.H, "bf16")
    want, scale = [], []
    for rows in _side_rows(w.R, "adjacent"):
        h = H[rows].reshape(-1, w.d)
        want.append(float(h.sum(axis=0) @ s) / (w.L * w.V))
        scale.append(_bound_terms(h.sum(axis=0), s, np.abs(h).sum(axis=0), S) / (w.L * w.V))
    _assert_close(got, want, scale)
