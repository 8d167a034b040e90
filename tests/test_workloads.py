"""Seeded input generator: shapes, length rules and the bf16 rounding it uses."""
import numpy as np
import pytest

from preference_alignment_b200 import workloads as WL


def test_bf16_round_to_nearest_even():
    # bf16 keeps 7 stored mantissa bits: the spacing just above 1.0 is 2^-7
    x = np.array([1.0, -2.0, 1.0 + 2**-7, 1.0 + 2**-8, 1.0 + 3 * 2**-8, 1.0 + 2**-9, 65504.0],
                 np.float32)
    bits = WL.bf16_bits_from_f32(x)
    # 1+2^-7 is exact; 1+2^-8 ties between 1 and 1+2^-7 -> even (1.0); 1+3*2^-8 ties between
    # 1+2^-7 and 1+2^-6 -> even (1+2^-6); 1+2^-9 rounds down; 65504 = 0x477FE000 rounds up
    assert list(bits) == [0x3F80, 0xC000, 0x3F81, 0x3F80, 0x3F82, 0x3F80, 0x4780]
    back = WL.bf16_bits_to_f32(bits)
    assert back[0] == 1.0 and back[2] == np.float32(1.0 + 2**-7)


def test_roundtrip_is_exact_for_bf16_values():
    rng = np.random.default_rng(0)
    b = rng.integers(0, 0x7F80, size=1000).astype(np.uint16)   # finite positives
    assert np.array_equal(WL.bf16_bits_from_f32(WL.bf16_bits_to_f32(b)), b)


def test_tiny_config_rules():
    w = WL.make_config("tiny")
    assert (w.R, w.L, w.d, w.V, w.dtype, w.layout) == (4, 32, 64, 1000, "f32", "adjacent")
    assert np.all((w.prompt_len >= 8) & (w.prompt_len <= 12))
    assert w.prompt_len[0] + w.completion_len[0] == 32           # row 0 has no pad
    assert w.completion_len[1] <= 3                              # row 1 is short
    assert np.all(w.completion_len >= 1)
    assert np.all(w.prompt_len + w.completion_len <= w.L)
    assert w.tokens.min() >= 0 and w.tokens.max() < w.V
    assert w.W_ref is not None and w.H.dtype == np.float32


def test_same_seed_same_inputs():
    a = WL.make_custom(R=4, L=20, d=8, V=30, seed=9)
    b = WL.make_custom(R=4, L=20, d=8, V=30, seed=9)
    for k in ("prompt_len", "completion_len", "tokens", "H", "W", "W_ref"):
        assert np.array_equal(getattr(a, k), getattr(b, k))


def test_custom_lengths_fit():
    w = WL.make_custom(R=9, L=50, d=8, V=30, seed=2, prompt_range=(1, 49), full_rows=2)
    assert np.all(w.prompt_len >= 1)
    assert np.all(w.prompt_len + w.completion_len <= 50)
    assert np.all(w.prompt_len[:2] + w.completion_len[:2] == 50)
