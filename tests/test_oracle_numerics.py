"""Pins for the oracle's bf16 round-to-nearest-even against torch's own conversion."""
import numpy as np
import torch

from oracle.numerics import bf16_bits_to_f32, f32_to_bf16_bits, round_bf16


def test_matches_torch_conversion_random():
    rng = np.random.default_rng(0)
    x = (rng.standard_normal(200000) * np.exp(rng.uniform(-20, 20, 200000))).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    assert np.array_equal(round_bf16(x), ref)


def test_exact_ties_round_to_even():
    # 1 + 2^-8 lies halfway between 1 and 1 + 2^-7: the even neighbour is 1.
    # 1 + 3*2^-8 lies halfway between 1 + 2^-7 (odd) and 1 + 2^-6 (even).
    x = np.array([1 + 2.0**-8, 1 + 3 * 2.0**-8, -(1 + 2.0**-8)], dtype=np.float32)
    assert np.array_equal(round_bf16(x), np.array([1.0, 1 + 2.0**-6, -1.0], dtype=np.float32))
    ref = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    assert np.array_equal(round_bf16(x), ref)


def test_bits_roundtrip():
    bits = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    f = bf16_bits_to_f32(bits)
    finite = np.isfinite(f)
    assert np.array_equal(f32_to_bf16_bits(f[finite]), bits[finite])
