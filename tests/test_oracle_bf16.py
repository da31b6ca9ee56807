"""Pins of the oracle's bf16 conversions (format definition + library routine)."""

import numpy as np
import pytest
import torch

from oracle import bf16_bits_to_f64, f64_to_bf16_bits, bf16_ulp_distance


def test_known_patterns():
    # Values fixed by the bfloat16 format: sign | 8-bit exponent | 7-bit mantissa.
    vals = np.array([1.0, -2.0, 0.5, 0.0, -0.0, 3.0, 1.0 / 3.0, 0.1])
    bits = f64_to_bf16_bits(vals)
    assert [hex(b) for b in bits] == [
        "0x3f80", "0xc000", "0x3f00", "0x0", "0x8000", "0x4040", "0x3eab", "0x3dcd"]
    assert bf16_bits_to_f64(np.array([0x3F80, 0xC040], dtype=np.uint16)).tolist() == [1.0, -3.0]


def test_ties_to_even():
    # 1 + 2^-8 lies halfway between 1 (mantissa ...0, even) and 1 + 2^-7 (odd).
    assert f64_to_bf16_bits(np.array([1.0 + 2.0 ** -8]))[0] == 0x3F80
    # 1 + 3*2^-8 lies halfway between 1 + 2^-7 (odd) and 1 + 2^-6 (even).
    assert f64_to_bf16_bits(np.array([1.0 + 3 * 2.0 ** -8]))[0] == 0x3F82
    # just above a tie rounds up
    assert f64_to_bf16_bits(np.array([1.0 + 2.0 ** -8 + 2.0 ** -30]))[0] == 0x3F81


def test_matches_torch_on_float32_values():
    rng = np.random.default_rng(7)
    x = (rng.standard_normal(20000) * 10.0 ** rng.integers(-20, 20, 20000)).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = f64_to_bf16_bits(x.astype(np.float64))
    assert np.array_equal(got, ref)


def test_roundtrip_exact():
    bits = np.arange(0, 0x7F80, 7, dtype=np.uint16)
    assert np.array_equal(f64_to_bf16_bits(bf16_bits_to_f64(bits)), bits)
    nb = bits | np.uint16(0x8000)
    assert np.array_equal(f64_to_bf16_bits(bf16_bits_to_f64(nb)), nb)


@pytest.mark.parametrize("a,b,d", [(0x3F80, 0x3F81, 1), (0x0000, 0x8000, 0),
                                   (0x0001, 0x8001, 2), (0x3F80, 0x4000, 128)])
def test_ulp_distance(a, b, d):
    assert int(bf16_ulp_distance(np.uint16(a), np.uint16(b))) == d
