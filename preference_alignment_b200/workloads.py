"""Seeded synthetic DPO head workloads.

This module only draws inputs: row lengths, target tokens, hidden states and
LM-head weights. It holds none of the method's arithmetic (no log-softmax, no
sums, no loss), so the CUDA path and the CPU oracle can both be fed from it
without sharing any computation.

Shapes follow the preference-batch layout of the pages: 2B rows, chosen and
rejected completions of the same prompt, each row = prompt | completion | pad
("DPO Training on GPU, in depth", section "What one DPO step computes"; the
concatenated [2B, L] batch of "Run Distributed Full-Model DPO with PyTorch
FSDP", Step 4). The head shape of the large cases is Llama 3.1 8B's
(d = 4096, V = 128,256; "DPO Training on GPU, in depth", section "Where the
memory goes for an 8B model").

Recipe (all draws from numpy PCG64(seed), in this order):
  1. prompt lengths P[R], then completion lengths C[R] (per-config rule);
  2. tokens [R, L] uniform on {0, ..., V-1} at every position;
  3. H [R, L, d] ~ N(0, 1);
  4. W [V, d] ~ N(0, 1/d);
  5. W_ref = W + N(0, sigma_ref^2) when the workload has a reference.
Normals are drawn in float32; bf16 workloads round them to bf16 with
round-to-nearest-even on the bit pattern (bf16_bits_from_f32 below).
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

SEED_BASE = 20261200


def bf16_bits_from_f32(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (round to nearest, ties to even); return the uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to float32 exactly."""
    b = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32)


def widen(arr: np.ndarray, dtype: str) -> np.ndarray:
    """Exact float64 view of a stored operand (bf16 bits or float32 values)."""
    if dtype == "bf16":
        return bf16_bits_to_f32(arr).astype(np.float64)
    return np.asarray(arr, dtype=np.float32).astype(np.float64)


@dataclasses.dataclass
class Workload:
    name: str
    R: int
    L: int
    d: int
    V: int
    dtype: str                 # "bf16" (uint16 bit arrays) or "f32" (float32 arrays)
    layout: str                # "halves" (chosen rows [0,B), rejected [B,2B)) or "adjacent"
    beta: float
    prompt_len: np.ndarray     # int32 [R]
    completion_len: np.ndarray # int32 [R]
    tokens: np.ndarray         # int32 [R, L]
    H: np.ndarray              # [R, L, d]
    W: np.ndarray              # [V, d]
    W_ref: Optional[np.ndarray]  # [V, d] or None (forward-only scoring workloads)
    seed: int = 0

    @property
    def B(self) -> int:
        return self.R // 2

    @property
    def n_scored(self) -> int:
        return int(self.completion_len.sum())


def _normal(rng, shape, std, dtype):
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return x


def encode(x: np.ndarray, dtype: str) -> np.ndarray:
    """Stored form of float32 draws: bf16 bit patterns (rounded) or float32 values."""
    return bf16_bits_from_f32(x) if dtype == "bf16" else np.ascontiguousarray(x, np.float32)


_encode = encode


def _draw_common(rng, R, L, d, V, dtype, ref_std, P, C, with_ref=True):
    tokens = rng.integers(0, V, size=(R, L), dtype=np.int64).astype(np.int32)
    H = _encode(_normal(rng, (R, L, d), 1.0, dtype), dtype)
    Wf = _normal(rng, (V, d), 1.0 / np.sqrt(d), dtype)
    W = _encode(Wf, dtype)
    W_ref = None
    if with_ref:
        noise = _normal(rng, (V, d), ref_std, dtype)
        # The reference is the policy's weights before rounding plus noise, then rounded.
        W_ref = _encode(Wf + noise, dtype)
    return tokens, H, W, W_ref


def _lengths_tiny(rng, R, L):
    P = rng.integers(8, 12 + 1, size=R)
    C = np.array([rng.integers(1, L - p + 1) for p in P])
    # Row 0 fills the row (no pad), row 1 has a short completion: both boundaries appear.
    C[0] = L - P[0]
    C[1] = min(C[1], 3)
    return P, C


def _lengths_small(rng, R, L):
    P = rng.integers(64, 256 + 1, size=R)
    C = np.array([rng.integers(32, L - p + 1) for p in P])
    return P, C


def _lengths_llama(rng, R, L):
    P = rng.integers(256, 1024 + 1, size=R)
    lo = int(np.ceil(0.95 * L))
    T = rng.integers(lo, L + 1, size=R)
    return P, T - P


def _lengths_offline(rng, R, L):
    P = rng.integers(128, 512 + 1, size=R)
    return P, L - P


def _lengths_long(rng, R, L):
    P = rng.integers(512, 3072 + 1, size=R)
    C = np.array([rng.integers(20, L - p + 1) for p in P])
    return P, C


# name -> (index, R, L, d, V, dtype, layout, ref_std, length rule, has_ref)
CONFIGS = {
    "tiny":    (1, 4, 32, 64, 1000, "f32", "adjacent", 0.01, _lengths_tiny, True),
    "small":   (2, 16, 512, 2048, 32000, "bf16", "halves", 0.01, _lengths_small, True),
    "llama8b": (3, 8, 2048, 4096, 128256, "bf16", "halves", 0.01, _lengths_llama, True),
    "offline": (4, 128, 1024, 4096, 128256, "bf16", "halves", 0.01, _lengths_offline, False),
    "long":    (5, 4, 4096, 2048, 151936, "bf16", "halves", 0.01, _lengths_long, True),
}

DESCRIPTIONS = {
    "tiny": "2 pairs -> 4 rows adjacent, L=32, d=64, V=1000, fp32",
    "small": "8 pairs -> 16 rows, L=512, d=2048, V=32000, bf16",
    "llama8b": "Llama-3.1-8B head: 4 pairs -> 8 rows, L=2048, d=4096, V=128256, bf16",
    "offline": "offline reference scoring: 64 pairs -> 128 rows, L=1024, d=4096, V=128256, bf16, fwd only",
    "long": "long ragged: 2 pairs -> 4 rows, L=4096, d=2048, V=151936, bf16",
}


def make_config(name: str, seed: Optional[int] = None, with_ref: Optional[bool] = None) -> Workload:
    idx, R, L, d, V, dtype, layout, ref_std, rule, has_ref = CONFIGS[name]
    seed = SEED_BASE + idx if seed is None else seed
    rng = np.random.Generator(np.random.PCG64(seed))
    P, C = rule(rng, R, L)
    want_ref = has_ref if with_ref is None else with_ref
    tokens, H, W, W_ref = _draw_common(rng, R, L, d, V, dtype, ref_std, P, C, with_ref=want_ref)
    return Workload(name, R, L, d, V, dtype, layout, 0.1, P.astype(np.int32), C.astype(np.int32),
                    tokens, H, W, W_ref, seed)


def make_custom(R: int, L: int, d: int, V: int, dtype: str = "bf16", layout: str = "halves",
                seed: int = 1, prompt_range=(1, None), min_completion: int = 0,
                ref_std: float = 0.01, with_ref: bool = True, beta: float = 0.1,
                full_rows: int = 0) -> Workload:
    """Small ragged workload for parity tests: prompt P ~ U{lo..hi}, completion C ~ U{min..L-P}.

    The first `full_rows` rows get C = L - P (completion runs to the end of the row).
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    lo, hi = prompt_range
    hi = L - 1 if hi is None else hi
    P = rng.integers(lo, hi + 1, size=R)
    C = np.array([rng.integers(min(min_completion, L - p), L - p + 1) for p in P])
    for i in range(min(full_rows, R)):
        C[i] = L - P[i]
    tokens, H, W, W_ref = _draw_common(rng, R, L, d, V, dtype, ref_std, P, C, with_ref=with_ref)
    return Workload("custom", R, L, d, V, dtype, layout, beta, P.astype(np.int32),
                    C.astype(np.int32), tokens, H, W, W_ref, seed)
