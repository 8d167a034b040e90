"""CUDA path vs the oracle at the full workload sizes, through the C ABI, in the
launch configuration bench.py times (default workspace, persistent CTA-pair grids).

- "small" (16 rows, d 2048, V 32,000): every output against the oracle.
- "llama8b", "offline", "long": outputs the oracle can compute one by one
  (sampled positions, including row and tile boundaries; one whole row or pair;
  sampled dH rows; for "long" also sampled dW rows), plus properties that hold at
  any size: dH is zero off the completion, the column sums of dW vanish
  (sum_v dz = 0), <dW, W> = <dH, H> (both equal sum dz * z), each sequence sum is
  the sum of its token log-probs, and no log-prob is positive.
"""
import numpy as np
import pytest

from oracle import dpo_oracle as O
from preference_alignment_b200 import libdpo
from preference_alignment_b200 import workloads as WL

from dpo_harness import (DeviceWorkload, TOL_GRAD, TOL_LOSS, TOL_TOK, assert_seq_close, np64,
                         rel_frob)

pytestmark = pytest.mark.gpu


class Widened:
    """float64 view of a bf16 weight, widened block by block on demand (saves host RAM)."""

    def __init__(self, W, dtype):
        self.Wbits, self.dtype, self.V = W, dtype, W.shape[0]
        self._full = None

    def __call__(self, a, b):
        return WL.widen(self.Wbits[a:b], self.dtype)

    def full(self):
        if self._full is None:
            self._full = WL.widen(self.Wbits, self.dtype)
        return self._full


def _sample_positions(w, n_random, seed):
    pos = O.scored_positions(w.prompt_len, w.completion_len, w.L)
    rng = np.random.default_rng(seed)
    idx = set(rng.choice(len(pos), size=min(n_random, len(pos)), replace=False).tolist())
    # row boundaries and tile boundaries of the packed order
    start = 0
    for c in w.completion_len:
        if c > 0:
            idx.update([start, start + int(c) - 1])
        start += int(c)
    for b in range(128, len(pos), 1280):
        idx.update([b - 1, b])
    # positions whose target falls in the last vocab tile (ragged when V % 256 != 0)
    last = (w.V - 1) // 256 * 256
    tail = [i for i, (r, t) in enumerate(pos) if w.tokens[r, t + 1] >= last]
    idx.update(tail[:8])
    return sorted(i for i in idx if i < len(pos)), pos


def _check_sampled_tokens(w, Wv, tok_gpu, lse_gpu, sample, pos):
    H = w.H
    rows = np.array([pos[i][0] for i in sample])
    ts = np.array([pos[i][1] for i in sample])
    h = WL.widen(H[rows, ts], w.dtype)
    lp, lse = O.position_logprobs(h, Wv, w.tokens[rows, ts + 1])
    err = np.abs(tok_gpu[rows, ts] - lp)
    assert err.max() <= TOL_TOK, f"token lp err {err.max()}"
    if lse_gpu is not None:
        assert np.abs(lse_gpu[np.array(sample)] - lse).max() <= TOL_TOK


def _check_properties_fwd(w, seq_gpu, tok_gpu):
    assert np.all(tok_gpu <= 1e-6)
    for r in range(w.R):
        p, c = w.prompt_len[r], w.completion_len[r]
        s = np.sum(tok_gpu[r, p - 1:p + c - 1], dtype=np.float64)
        assert abs(seq_gpu[r] - s) <= 1e-4 * max(1.0, abs(s))
        mask = np.ones(w.L, bool)
        mask[p - 1:p + c - 1] = False
        assert np.all(tok_gpu[r, mask] == 0.0)


def _check_properties_bwd(w, dH, dW, H_dev, W_dev):
    import torch
    gH = dH.cpu()
    for r in range(w.R):
        p, c = w.prompt_len[r], w.completion_len[r]
        mask = torch.ones(w.L, dtype=torch.bool)
        mask[p - 1:p + c - 1] = False
        assert torch.all(gH[r][mask] == 0.0)
    colsum = dW.double().sum(dim=0)
    fro = torch.linalg.norm(dW.double())
    assert float(torch.linalg.norm(colsum) / fro) <= TOL_GRAD
    a = float((dW.double() * W_dev.double()).sum())
    b = float((dH.double() * H_dev.double()).sum())
    assert abs(a - b) <= TOL_GRAD * max(abs(a), abs(b), 1e-30)


def _check_sampled_dH(w, Wv, dH_gpu, coef, sample, pos):
    W64 = Wv.full()
    got, want = [], []
    for i in sample:
        r, t = pos[i]
        h = WL.widen(w.H[r, t], w.dtype)
        want.append(O.position_grad_h(h, W64, w.tokens[r, t + 1], coef[r]))
        got.append(dH_gpu[r, t])
    assert rel_frob(np.array(got), np.array(want)) <= TOL_GRAD


# ---------------------------------------------------------------------- small: full parity
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
    assert_seq_close(np64(pol), op["seq_logp"])
    assert_seq_close(np64(ref), orf["seq_logp"])
    assert abs(out["loss"].item() - ol["loss"]) <= TOL_LOSS          # end to end
    np.testing.assert_allclose(np64(out["margins"]), ol["margins"], atol=5e-3)
    assert out["accuracy"].item() == pytest.approx(ol["accuracy"], abs=1e-7)

    dH, dW = dw.backward(lse, torch.from_numpy(ol["row_coef"].astype(np.float32)).cuda())
    assert libdpo.check() == libdpo.OK
    oH, oW = O.backward(H64, W64, w.tokens, w.prompt_len, w.completion_len, ol["row_coef"])
    assert rel_frob(np64(dH), oH) <= TOL_GRAD
    assert rel_frob(np64(dW), oW) <= TOL_GRAD


# ---------------------------------------------------------------------- large: sampled
def _large_forward_backward(name, seed, backward=True, dW_rows=0):
    import torch
    w = WL.make_config(name)
    dw = DeviceWorkload(w)
    Wv = Widened(w.W, w.dtype)
    sample, pos = _sample_positions(w, 48, seed)

    seq, tok, lse = dw.forward(dw.W, want_grad=backward)
    assert libdpo.check() == libdpo.OK
    seq_np, tok_np = np64(seq), np64(tok)
    _check_properties_fwd(w, seq_np, tok_np)
    _check_sampled_tokens(w, Wv, tok_np, np64(lse) if backward else None, sample, pos)

    # one whole row against the oracle: the row with the fewest scored positions
    r = int(np.argmin(np.where(w.completion_len > 0, w.completion_len, 1 << 30)))
    sub = O.seq_logprobs(WL.widen(w.H[r:r + 1], w.dtype), Wv.full(), w.tokens[r:r + 1],
                         w.prompt_len[r:r + 1], w.completion_len[r:r + 1])
    assert_seq_close(seq_np[r:r + 1], sub["seq_logp"])

    if not backward:
        return w
    # the loss kernel on the full-size sums, against the oracle's loss on the same sums
    ref, _, _ = dw.forward(dw.W_ref, want_grad=False)
    out = dw.loss(seq, ref)
    ol = O.dpo_loss(np64(seq), np64(ref), w.beta, w.layout)
    assert abs(out["loss"].item() - ol["loss"]) <= TOL_LOSS
    coef = np.random.default_rng(seed).normal(0, 0.02, size=w.R).astype(np.float32)
    dH, dW = dw.backward(lse, torch.from_numpy(coef).cuda())
    assert libdpo.check() == libdpo.OK
    _check_properties_bwd(w, dH, dW, dw.H.float(), dw.W.float())
    _check_sampled_dH(w, Wv, np64(dH), coef.astype(np.float64), sample[:40], pos)
    if dW_rows:
        # dW[v] = sum_t dz[t, v] h_t needs softmax(z_t)[v] at every scored position: the
        # oracle's full forward gives lse_t, then the chosen vocab rows are summed exactly
        H64 = WL.widen(w.H, w.dtype)
        full = O.seq_logprobs(H64, Wv.full(), w.tokens, w.prompt_len, w.completion_len)
        rows = np.array([p[0] for p in pos])
        ts = np.array([p[1] for p in pos])
        hs = H64[rows, ts]
        ys = w.tokens[rows, ts + 1]
        vs = np.unique(np.concatenate([ys[:dW_rows // 2],
                                       np.random.default_rng(seed).integers(0, w.V, dW_rows // 2)]))
        z = hs @ Wv.full()[vs].T                              # [Nc, |vs|]
        p = np.exp(z - full["lse"][:, None])
        dz = -p
        for j, v in enumerate(vs):
            dz[ys == v, j] += 1.0
        dz *= coef.astype(np.float64)[rows][:, None]
        want = dz.T @ hs
        assert rel_frob(np64(dW[torch.from_numpy(vs).cuda()]), want) <= TOL_GRAD
    return w


def test_llama8b_head_sampled():
    _large_forward_backward("llama8b", seed=3)


def test_offline_scoring_sampled():
    _large_forward_backward("offline", seed=4, backward=False)


def test_long_ragged_sampled():
    _large_forward_backward("long", seed=5, dW_rows=16)
