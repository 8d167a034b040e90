"""Plain CPU float64 oracle for the DPO head path.

TEST INFRASTRUCTURE ONLY. Nothing in the product path may import or call this
module: only the tests, `__graft_entry__.smoke()` and the CPU-baseline leg of
`bench.py` use it. It shares no code with the CUDA library; both sides are fed
the same seeded arrays and nothing else.

What it computes, step by step, in the order of the pages:

* Sequence log-probability of a completion = sum over the completion tokens of
  log p(token | everything before it), with the prompt kept as conditioning
  ("DPO Training on GPU, in depth", section "What one DPO step computes").
* Position t predicts token t+1: logits[:, :-1] pair with labels[:, 1:] and
  mask[:, 1:]; log-softmax over the full vocabulary, then the target is picked
  and multiplied by the completion mask ("DPO Training on GPU, in depth",
  section "A training configuration that fits", the hand-written
  sequence_logps / _chunk_logps). Positions are processed in chunks of 256 as
  that section does; each chunk is a plain matrix product.
* DPO loss: -log sigmoid(beta * [(pi_c - ref_c) - (pi_r - ref_r)]), averaged over
  pairs; rewards = beta * log-ratio; margin = r_c - r_r; per-pair gradient
  weight sigmoid(-margin); accuracy = fraction of pairs with margin > 0
  ("DPO Training on GPU, in depth", sections "What one DPO step computes" and
  "A worked example of the numbers", and dpo_step in "A training configuration
  that fits").
* Logits-mean metrics: the mean of the chosen rows' logits and of the rejected
  rows' logits over every position and vocabulary entry ("Run Distributed
  Full-Model DPO with PyTorch FSDP", Step 4 and "What to Watch Out For").
* Backward of the loss through the sequence sums to the LM-head input H and
  weight W: dL/dz[t, v] = dL/dS_r * (onehot(y_t)[v] - softmax(z_t)[v]),
  dH[t] = dZ[t] . W, dW = sum_t dZ[t]^T h_t (chain rule on the definitions
  above; the pages run it as loss.backward()).

Readings where the pages leave a step open (each is listed in the design notes):
* row r with prompt length P_r and completion length C_r scores positions
  t in [P_r - 1, P_r + C_r - 1); P_r >= 1;
* the batch loss is the mean over pairs; accuracy uses the strict margin > 0;
* returned margins include beta; weights are sigmoid(-margin) without beta/B;
* row_coef[r] = d(grad_scale * loss) / d seq_logp[r].

Every function here is pinned by tests in tests/test_oracle_pins.py against
values that do not come from this module: the pages' worked example, ln 2 at
policy == reference, closed forms, 50-digit brute force, finite differences and
invariants of the mathematics.
"""
from __future__ import annotations

import decimal
import math

import numpy as np

CHUNK = 256  # positions per chunk, as the pages' hand-written loss does


# --------------------------------------------------------------------------------------
# Scored positions
# --------------------------------------------------------------------------------------
def scored_positions(prompt_len, completion_len, L):
    """List of (row, position) pairs that are scored, in row order.

    Completion tokens are indices [P, P + C) of the row; token j is predicted by
    position j - 1, so the scored positions are [P - 1, P + C - 1).
    """
    out = []
    for r, (p, c) in enumerate(zip(prompt_len, completion_len)):
        p, c = int(p), int(c)
        if p < 1 or c < 0 or p + c > L:
            raise ValueError(f"row {r}: prompt {p} completion {c} does not fit length {L}")
        for t in range(p - 1, p + c - 1):
            out.append((r, t))
    return out


# --------------------------------------------------------------------------------------
# Per-position log-probabilities
# --------------------------------------------------------------------------------------
def position_logprobs(h, W, targets, vocab_chunk=None):
    """log p(target) under softmax(h . W^T) for a set of positions.

    h: [n, d] float64, W: [V, d] (float64, or a callable giving float64 row blocks
    W[a:b] when the weight is too large to widen at once), targets: [n] ints.
    Returns (lp [n], lse [n]) with lse = log sum_v exp(z_v), z = h . W^T.
    """
    h = np.asarray(h, dtype=np.float64)
    n = h.shape[0]
    if callable(W):
        V = W.V
        z = np.empty((n, V), dtype=np.float64)
        step = vocab_chunk or 8192
        for a in range(0, V, step):
            b = min(V, a + step)
            z[:, a:b] = h @ W(a, b).T
    else:
        z = h @ np.asarray(W, dtype=np.float64).T
    m = z.max(axis=1)
    lse = m + np.log(np.exp(z - m[:, None]).sum(axis=1))
    zy = z[np.arange(n), np.asarray(targets, dtype=np.int64)]
    return zy - lse, lse


def seq_logprobs(H, W, tokens, prompt_len, completion_len):
    """Sequence log-prob sums per row, plus per-token values and the log-sum-exp.

    H: [R, L, d] float64, W: [V, d] float64, tokens: [R, L] ints.
    Returns dict with
      seq_logp [R]      sum over the row's scored positions (math.fsum),
      tok_logp [R, L]   log-prob at scored positions, 0 elsewhere,
      lse [Nc]          log-sum-exp per scored position in row order,
      positions         the scored (row, position) list.
    """
    R, L, d = H.shape
    pos = scored_positions(prompt_len, completion_len, L)
    tok_logp = np.zeros((R, L), dtype=np.float64)
    lse_all = np.zeros(len(pos), dtype=np.float64)
    for s in range(0, len(pos), CHUNK):
        chunk = pos[s:s + CHUNK]
        rows = np.array([r for r, _ in chunk])
        ts = np.array([t for _, t in chunk])
        lp, lse = position_logprobs(H[rows, ts], W, tokens[rows, ts + 1])
        tok_logp[rows, ts] = lp
        lse_all[s:s + len(chunk)] = lse
    seq = np.array([
        math.fsum(tok_logp[r, int(p) - 1:int(p) + int(c) - 1])
        for r, (p, c) in enumerate(zip(prompt_len, completion_len))
    ], dtype=np.float64)
    return {"seq_logp": seq, "tok_logp": tok_logp, "lse": lse_all, "positions": pos}


# --------------------------------------------------------------------------------------
# Loss
# --------------------------------------------------------------------------------------
def pair_rows(B, layout):
    """(chosen_row, rejected_row) for each pair i under a row layout."""
    if layout == "halves":       # chosen rows first, then rejected rows
        return [(i, B + i) for i in range(B)]
    if layout == "adjacent":     # chosen and rejected of a pair next to each other
        return [(2 * i, 2 * i + 1) for i in range(B)]
    raise ValueError(layout)


def softplus(x):
    """log(1 + e^x), evaluated without overflow."""
    return max(x, 0.0) + math.log1p(math.exp(-abs(x)))


def sigmoid(x):
    """1 / (1 + e^-x), evaluated without overflow."""
    if x >= 0:
        return 1.0 / (1.0 + math.exp(-x))
    e = math.exp(x)
    return e / (1.0 + e)


def dpo_loss(pol, ref, beta, layout="halves", grad_scale=1.0, completion_len=None,
             normalize=False, nll_weight=0.0, pairs_total=None, nll_tokens_total=None):
    """Sigmoid DPO loss and its metrics, from policy and reference sequence sums.

    pol, ref: [2B] sequence log-prob sums in the row layout. The log-ratios are
    formed first, then their difference, as the pages' dpo_step does.

    Variants ("Run Distributed Full-Model DPO with PyTorch FSDP", Step 4: sums let
    the loss use length-normalised or sum-based rewards; "DPO Training on GPU, in
    depth", failure modes: length-normalised variants and an added SFT term; the
    video transcript: total loss = DPO loss + lambda * NLL on the chosen responses):
      normalize   use S_r / C_r (the average completion log-prob; 0 for C_r = 0)
                  for policy and reference alike;
      nll_weight  lambda: add lambda * NLL, the standard language-modelling loss on
                  the chosen completions, read as the mean over all their tokens:
                  NLL = -(sum of chosen S_r) / (sum of chosen C_r), from raw sums.
    completion_len [2B] is needed by either variant.

    Data-parallel shares ("Run Distributed Full-Model DPO with PyTorch FSDP", Step 1:
    every rank holds part of the global batch): with pairs_total = B_g the batch
    means (loss, accuracy, row_coef) divide by B_g instead of this call's B, and
    with nll_tokens_total = N_g the NLL divides by N_g; the outputs are then this
    part's share of the whole batch's values, and the shares of a partition of the
    batch add up to the values of the whole.

    Reference-free objective (ref=None; "Run Distributed Full-Model DPO with PyTorch
    FSDP", "Where to Go Next": it skips the frozen reference model; the formula is
    not given there): the reference sums are read as 0, so the log-ratios are the
    policy's own (normalised) sums, rewards beta * pi and margin beta * (pi_c - pi_r).
    """
    pol = [float(x) for x in pol]
    R = len(pol)
    ref = [0.0] * R if ref is None else [float(x) for x in ref]
    if len(ref) != R:
        raise ValueError("policy and reference sums differ in length")
    if R % 2:
        raise ValueError("odd number of rows")
    B = R // 2
    Bdiv = B if pairs_total is None else int(pairs_total)
    C = None if completion_len is None else [int(c) for c in completion_len]
    if (normalize or nll_weight) and C is None:
        raise ValueError("completion lengths are needed for the loss variants")
    scale = [1.0] * R                      # d(value used in the loss)/d(raw sum)
    if normalize:
        scale = [1.0 / c if c > 0 else 0.0 for c in C]
    pv = [pol[r] * scale[r] for r in range(R)]
    rv = [ref[r] * scale[r] for r in range(R)]
    margins, rc, rr, w, losses = [], [], [], [], []
    coef = [0.0] * R
    for i, (c, r) in enumerate(pair_rows(B, layout)):
        rho_c = pv[c] - rv[c]
        rho_r = pv[r] - rv[r]
        m = beta * (rho_c - rho_r)
        margins.append(m)
        rc.append(beta * rho_c)
        rr.append(beta * rho_r)
        wi = sigmoid(-m)
        w.append(wi)
        losses.append(softplus(-m))          # -log sigmoid(m)
        # d softplus(-m)/dm = -sigmoid(-m); dm/dpol[c] = beta, dm/dpol[r] = -beta
        coef[c] = -grad_scale * beta * wi / Bdiv * scale[c]
        coef[r] = +grad_scale * beta * wi / Bdiv * scale[r]
    loss = math.fsum(losses) / Bdiv
    nll = 0.0
    if nll_weight:
        chosen = [c for c, _ in pair_rows(B, layout)]
        ntok = sum(C[c] for c in chosen) if nll_tokens_total is None else int(nll_tokens_total)
        if ntok > 0:
            nll = -math.fsum(pol[c] for c in chosen) / ntok
            for c in chosen:
                coef[c] += -grad_scale * nll_weight / ntok
        loss = loss + nll_weight * nll
    return {
        "loss": loss,
        "accuracy": sum(1.0 for m in margins if m > 0) / Bdiv,
        "margins": np.array(margins),
        "chosen_rewards": np.array(rc),
        "rejected_rewards": np.array(rr),
        "weights": np.array(w),
        "row_coef": np.array(coef),
        "losses": np.array(losses),
        "nll": nll,
    }


# --------------------------------------------------------------------------------------
# Backward
# --------------------------------------------------------------------------------------
def backward(H, W, tokens, prompt_len, completion_len, row_coef):
    """Gradients of sum_r row_coef[r] * seq_logp[r] w.r.t. H and W.

    For each scored position t of row r: dz = row_coef[r] * (onehot(y) - softmax(z)),
    dH[r, t] = dz . W, dW += outer(dz, h_t). Unscored positions get dH = 0.
    Returns (dH [R, L, d], dW [V, d]) in float64.
    """
    R, L, d = H.shape
    W = np.asarray(W, dtype=np.float64)
    V = W.shape[0]
    pos = scored_positions(prompt_len, completion_len, L)
    dH = np.zeros_like(H, dtype=np.float64)
    dW = np.zeros((V, d), dtype=np.float64)
    for s in range(0, len(pos), CHUNK):
        chunk = pos[s:s + CHUNK]
        rows = np.array([r for r, _ in chunk])
        ts = np.array([t for _, t in chunk])
        h = H[rows, ts]                          # [n, d]
        z = h @ W.T                              # [n, V]
        m = z.max(axis=1, keepdims=True)
        p = np.exp(z - m)
        p /= p.sum(axis=1, keepdims=True)        # softmax
        dz = -p
        dz[np.arange(len(chunk)), tokens[rows, ts + 1]] += 1.0
        dz *= np.asarray(row_coef, dtype=np.float64)[rows][:, None]
        dH[rows, ts] = dz @ W
        dW += dz.T @ h
    return dH, dW


def position_grad_h(h, W, target, coef):
    """dH row of one scored position: coef * (W[y] - softmax(z) . W); W float64 [V, d]."""
    z = W @ np.asarray(h, dtype=np.float64)
    p = np.exp(z - z.max())
    p /= p.sum()
    return coef * (W[int(target)] - p @ W)


# --------------------------------------------------------------------------------------
# Logits-mean metrics
# --------------------------------------------------------------------------------------
def logits_mean(H, W, layout="halves"):
    """Mean of the logits over the chosen rows and over the rejected rows.

    The torchtune DPO loop of "Run Distributed Full-Model DPO with PyTorch FSDP"
    splits the model's logits for the concatenated batch into the chosen and the
    rejected halves (Step 4, concatenated_forward: every position of every row,
    prompt and padding included, over the whole vocabulary) and logs their means as
    policy_chosen_logits_mean and policy_rejected_logits_mean ("What to Watch Out
    For"). Here the logits z = h_t . W^T of every position t of every row on one
    side are formed chunk by chunk and averaged over rows x positions x vocabulary;
    the layout says which rows are chosen (pair_rows). H: [R, L, d], W: [V, d].
    Returns (chosen_mean, rejected_mean).
    """
    H = np.asarray(H, dtype=np.float64)
    W = np.asarray(W, dtype=np.float64)
    R, L, _ = H.shape
    V = W.shape[0]
    B = R // 2
    means = []
    for side in (0, 1):
        sums = []
        for pair in pair_rows(B, layout):
            r = pair[side]
            for t0 in range(0, L, CHUNK):
                Z = H[r, t0:t0 + CHUNK] @ W.T
                sums.append(math.fsum(Z.ravel()))
        means.append(math.fsum(sums) / (B * L * V))
    return means[0], means[1]


# --------------------------------------------------------------------------------------
# 50-digit brute force for tiny problems
# --------------------------------------------------------------------------------------
def logprob_bruteforce(h, W, target, digits=50):
    """log p(target) for one position, every step in `decimal` arithmetic.

    z_v = sum_k h_k W[v, k] exactly (inputs are binary floats, so exact in
    decimal), then log(exp(z_y) / sum_v exp(z_v)). Meant for V <= 8, d <= 4.
    """
    ctx = decimal.Context(prec=digits)
    D = decimal.Decimal
    z = []
    for v in range(len(W)):
        acc = D(0)
        for k in range(len(h)):
            acc = ctx.add(acc, ctx.multiply(D(float(h[k])), D(float(W[v][k]))))
        z.append(acc)
    tot = D(0)
    for zv in z:
        tot = ctx.add(tot, ctx.exp(zv))
    return ctx.subtract(z[int(target)], ctx.ln(tot))
