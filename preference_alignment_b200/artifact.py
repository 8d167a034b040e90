"""Offline reference scores: store them once, check them before every use.

The reference model is frozen, so its per-row completion log-prob sums can be
computed once (dpo_seq_logprobs without grad state) and read back by every later
run ("DPO Training on GPU, in depth", "Four ways to host the reference model",
precomputed log-probabilities; Megatron-Bridge PR 6092, "Why the reference is
scored offline"). Following the PR:
  - scores are stored per pair (chosen and rejected sums) and joined back to the
    pairs by index;
  - the sums carry no beta, so one scoring run serves every beta;
  - a metadata record is written beside them, and loading refuses any mismatch
    with what the caller expects, because a stale or mis-scored artifact would not
    crash anything, it would only bias every margin.
The metadata always holds the head shape (d, V, L), the dtype, the library
version and the 64-bit fingerprint of the reference weights (dpo_fingerprint);
callers add their own keys (dataset, split, tokenizer, ...).

Files: <dir>/ref_logprobs.jsonl (one {"pair", "chosen", "rejected"} per line) and
<dir>/scoring_metadata.json.
"""
from __future__ import annotations

import json
import os
from typing import Dict, Optional

import numpy as np

SCORES = "ref_logprobs.jsonl"
META = "scoring_metadata.json"


class ArtifactMismatch(RuntimeError):
    pass


def pair_rows(B: int, layout: str):
    if layout == "halves":
        return [(i, B + i) for i in range(B)]
    if layout == "adjacent":
        return [(2 * i, 2 * i + 1) for i in range(B)]
    raise ValueError(layout)


def save(path: str, seq_logp, layout: str, meta: Dict, pair_offset: int = 0, append: bool = False):
    """Write the per-pair sums of one batch (rows in `layout`) and the metadata record.

    pair_offset numbers the pairs of this batch in the dataset; with append=True a
    later batch is added to the same artifact (the metadata must be identical)."""
    os.makedirs(path, exist_ok=True)
    seq = np.asarray(seq_logp, dtype=np.float64)
    if seq.ndim != 1 or seq.size % 2:
        raise ValueError("seq_logp must hold 2B row sums")
    meta_path = os.path.join(path, META)
    if append and os.path.exists(meta_path):
        check(path, meta)
    else:
        with open(meta_path, "w") as f:
            json.dump(meta, f, indent=1, sort_keys=True)
    with open(os.path.join(path, SCORES), "a" if append else "w") as f:
        for i, (c, r) in enumerate(pair_rows(seq.size // 2, layout)):
            f.write(json.dumps({"pair": pair_offset + i, "chosen": float(seq[c]),
                                "rejected": float(seq[r])}) + "\n")


def check(path: str, expect: Dict):
    """Raise ArtifactMismatch unless every expected key matches the stored metadata."""
    with open(os.path.join(path, META)) as f:
        stored = json.load(f)
    bad = {k: (stored.get(k), v) for k, v in expect.items() if stored.get(k) != v}
    if bad:
        raise ArtifactMismatch("reference scores were produced under a different setup: " +
                               ", ".join(f"{k}: stored {a!r}, expected {b!r}" for k, (a, b) in
                                         sorted(bad.items())))
    return stored


def load(path: str, expect: Dict, pairs: Optional[np.ndarray] = None, layout: str = "halves"):
    """Check the metadata, then return the [2B] reference sums of the given pairs in `layout`."""
    check(path, expect)
    table = {}
    with open(os.path.join(path, SCORES)) as f:
        for line in f:
            if line.strip():
                rec = json.loads(line)
                table[int(rec["pair"])] = (rec["chosen"], rec["rejected"])
    idx = sorted(table) if pairs is None else [int(p) for p in pairs]
    missing = [p for p in idx if p not in table]
    if missing:
        raise ArtifactMismatch(f"pairs missing from the artifact: {missing[:8]}")
    B = len(idx)
    out = np.zeros(2 * B, dtype=np.float64)
    for i, (c, r) in enumerate(pair_rows(B, layout)):
        out[c], out[r] = table[idx[i]]
    return out


def metadata(d: int, V: int, L: int, dtype: str, weights_fingerprint: int, lib_version: int,
             **extra) -> Dict:
    """The metadata record: head shape, dtype, weight fingerprint, library version + extras."""
    m = {"d": int(d), "V": int(V), "L": int(L), "dtype": dtype,
         "weights_fingerprint": f"{int(weights_fingerprint) & ((1 << 64) - 1):016x}",
         "libdpo_version": int(lib_version)}
    m.update(extra)
    return m
