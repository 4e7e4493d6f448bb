"""Pins of the oracle's bfloat16 rounder.

Two independent anchors: torch's float32 -> bfloat16 conversion (a library
routine that rounds to nearest, ties to even) on values spanning the whole
exponent range, and hand-worked IEEE cases (ties, subnormals, overflow).
"""
import numpy as np
import torch

from oracle import bf16_round, bf16_bits, bf16_from_bits, bf16_ulp


def _torch_bf16(x32):
    return torch.from_numpy(x32).to(torch.bfloat16).to(torch.float64).numpy()


def test_matches_torch_on_random_float32():
    rng = np.random.default_rng(0)
    mant = rng.uniform(1.0, 2.0, 200_000)
    expo = rng.integers(-149, 128, 200_000)
    sign = rng.choice([-1.0, 1.0], 200_000)
    x = (sign * np.ldexp(mant, expo)).astype(np.float32)
    x = x[np.isfinite(x)]
    ours = bf16_round(x.astype(np.float64))
    ref = _torch_bf16(x)
    assert np.array_equal(ours, ref)


def test_matches_torch_on_exact_ties():
    # every float32 exactly halfway between two bfloat16 neighbours
    rng = np.random.default_rng(1)
    hi = rng.integers(0, 0x7F7F, 100_000, dtype=np.uint32)          # finite bf16 patterns
    x = ((hi << 16) | 0x8000).view(np.float32)                        # halfway to the next
    x = np.concatenate([x, -x])
    assert np.array_equal(bf16_round(x.astype(np.float64)), _torch_bf16(x))


def test_hand_worked_cases():
    two = 2.0
    assert bf16_round(1 + two ** -8) == 1.0                     # tie -> even (down)
    assert bf16_round(1 + 3 * two ** -8) == 1 + two ** -6        # tie -> even (up)
    assert bf16_round(1 + two ** -8 + two ** -30) == 1 + two ** -7   # just above the tie
    assert bf16_round(-(1 + two ** -8)) == -1.0
    assert bf16_round(3.0) == 3.0 and bf16_round(0.0) == 0.0
    assert np.signbit(bf16_round(-0.0))
    bf16_max = (2 - two ** -7) * two ** 127
    assert bf16_round(bf16_max) == bf16_max
    assert np.isinf(bf16_round(two ** 128 - two ** 119))         # tie at the top -> inf
    assert bf16_round(two ** 128 - two ** 119 - two ** 100) == bf16_max
    assert bf16_round(two ** -133) == two ** -133                # smallest subnormal
    assert bf16_round(two ** -134) == 0.0                        # tie between 0 and it -> 0
    assert bf16_round(3 * two ** -135) == two ** -133
    assert bf16_round(1.5 * two ** -133) == 2 * two ** -133      # tie -> even (up)
    assert np.isnan(bf16_round(np.nan)) and bf16_round(-np.inf) == -np.inf


def test_bits_roundtrip_and_ulp():
    v = bf16_round(np.array([1.0, -2.5, 3.140625, 1e-3, 6e4]))
    assert np.array_equal(bf16_from_bits(bf16_bits(v)), v)
    assert bf16_bits(np.array([1.0]))[0] == 0x3F80
    assert bf16_ulp(1.0) == 2.0 ** -7 and bf16_ulp(1.99) == 2.0 ** -7 and bf16_ulp(2.0) == 2.0 ** -6
