"""Pins of the oracle's number formats against definitions that do not come
from the oracle itself: library casts (torch), exhaustive bit-field decoding,
brute-force nearest-value search and hand-worked values.

Formats: NVFP4 = E2M1 values in groups of 16 with FP8 (E4M3) scales, INT4 in
groups of 64 with 16-bit scales (SOTA-314 practice page, "Do this").
"""
import itertools
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import svdq_oracle as o


# ---------------------------------------------------------------- BF16

def test_bf16_round_matches_torch_cast_on_float32():
    rng = np.random.default_rng(1)
    x = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * 10.0 ** rng.integers(-30, 30, 20000),
        # exact ties: a float32 with the 9th significant bit set and nothing below
        (np.arange(1, 2000, dtype=np.float32) * 2 + 1) * np.float32(2.0 ** -9) + np.float32(1.0),
        np.array([0.0, -0.0, 1e-40, -1e-40, 3.0e38], dtype=np.float32),
    ]).astype(np.float32)
    want = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    got = o.bf16_round(x.astype(np.float64))
    np.testing.assert_array_equal(got, want)


def test_bf16_round_single_rounding_from_float64():
    # 1 + 2^-8 + 2^-30: above the tie, so it rounds up; a float32 detour would
    # first drop 2^-30 and then round the exact tie down to 1.
    x = 1.0 + 2.0 ** -8 + 2.0 ** -30
    assert o.bf16_round(x) == 1.0 + 2.0 ** -7
    assert o.bf16_round(1.0 + 2.0 ** -8) == 1.0            # tie -> even
    assert o.bf16_round(1.0 + 3 * 2.0 ** -8) == 1.0 + 2.0 ** -6


# ---------------------------------------------------------------- E4M3

def _e4m3_bitfield(b):
    """Decode from the E4M3 bit-field definition with exact rationals."""
    s, e, m = b >> 7, (b >> 3) & 0xF, b & 7
    if e == 15 and m == 7:
        return None
    v = Fraction(m, 8) * Fraction(2) ** -6 if e == 0 else (1 + Fraction(m, 8)) * Fraction(2) ** (e - 7)
    return -v if s else v


def test_e4m3_decode_all_bytes():
    codes = np.arange(256, dtype=np.uint8)
    lib = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = o.e4m3_decode(codes)
    for b in range(256):
        ref = _e4m3_bitfield(b)
        if ref is None:
            assert np.isnan(ours[b]) and np.isnan(lib[b])
        else:
            assert ours[b] == float(ref) == lib[b], b


def test_e4m3_encode_roundtrip_all_finite_nonnegative():
    for b in range(127):                                 # 0x00..0x7E, sign 0, finite
        v = o.e4m3_decode(b)
        assert o.e4m3_encode(v) == b
        assert o.e4m3_round_satfinite(v) == v


def test_e4m3_round_matches_torch_cast_in_range():
    rng = np.random.default_rng(2)
    finite = o.e4m3_decode(np.arange(127))
    mids = (finite[1:] + finite[:-1]) / 2                # exact ties
    x = np.concatenate([rng.uniform(0, 448, 20000), rng.uniform(0, 2.0 ** -5, 5000),
                        10.0 ** rng.uniform(-4, 2.6, 20000), mids, finite]).astype(np.float32)
    x = x[x <= 448]
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = o.e4m3_round_satfinite(x.astype(np.float64))
    np.testing.assert_array_equal(got, want)


def test_e4m3_saturates_at_448():
    got = o.e4m3_round_satfinite(np.array([448.0, 463.9, 464.0, 470.0, 1e6]))
    np.testing.assert_array_equal(got, [448.0] * 5)
    assert o.e4m3_encode(448.0) == 0x7E


# ---------------------------------------------------------------- E2M1

def test_e2m1_decode_bitfield():
    # E2M1: 1 sign, 2 exponent bits (bias 1), 1 mantissa bit; exponent 0 is subnormal.
    for c in range(16):
        s, e, m = c >> 3, (c >> 1) & 3, c & 1
        v = Fraction(m, 2) if e == 0 else (1 + Fraction(m, 2)) * Fraction(2) ** (e - 1)
        assert o.e2m1_decode(c) == float(-v if s else v)


def test_e2m1_encode_brute_force_nearest_even():
    grid = [float(o.e2m1_decode(c)) for c in range(8)]
    rng = np.random.default_rng(3)
    vals = np.concatenate([rng.uniform(-8, 8, 20000), np.arange(-70, 71) / 10.0,
                           np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25, -5.0, 0.0, -0.0])])
    got = o.e2m1_encode(vals)
    for v, g in zip(vals, got):
        a = min(abs(v), 6.0)
        d = [abs(a - x) for x in grid]
        best = min(d)
        cands = [c for c in range(8) if d[c] == best]
        mag = cands[0] if len(cands) == 1 else [c for c in cands if c % 2 == 0][0]
        want = mag | (8 if np.signbit(v) else 0)
        assert g == want, (v, g, want)


def test_e2m1_ties_hand_worked():
    # the grid's midpoints go to the even code
    got = o.e2m1_encode([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 7.0, -0.1])
    assert list(got) == [0, 2, 2, 4, 4, 6, 6, 7, 8]


def test_pack_nibbles_even_low():
    codes = np.array([[0x1, 0x2, 0xF, 0x0, 0x8, 0x7]], dtype=np.uint8)
    assert list(o.pack_nibbles(codes)[0]) == [0x21, 0x0F, 0x78]
    np.testing.assert_array_equal(o.unpack_nibbles(o.pack_nibbles(codes)), codes)


def test_int4_nibbles_twos_complement():
    c = np.arange(-7, 8)
    np.testing.assert_array_equal(o.int4_decode(o.int4_nibbles(c)), c)
    assert o.int4_nibbles(np.array([-1]))[0] == 0xF


# ---------------------------------------------------------------- constants

def test_float32_reciprocal_constants_are_correctly_rounded():
    # fp32(1/6) and fp32(1/7) as the oracle forms them equal the nearest
    # float32 to the exact rationals.
    for d in (6, 7):
        c = np.float32(1.0 / d)
        exact = Fraction(1, d)
        below = np.nextafter(c, np.float32(0))
        above = np.nextafter(c, np.float32(1))
        assert abs(Fraction(float(c)) - exact) <= abs(Fraction(float(below)) - exact)
        assert abs(Fraction(float(c)) - exact) <= abs(Fraction(float(above)) - exact)


def test_pow2_exponent_ceil():
    assert o.pow2_exponent_ceil(1.0) == 0
    assert o.pow2_exponent_ceil(1.0000001) == 1
    assert o.pow2_exponent_ceil(0.5) == -1
    assert o.pow2_exponent_ceil(0.75) == 0
    assert o.pow2_exponent_ceil(2688.0) == 12
    for x in 10.0 ** np.linspace(-20, 20, 301):
        e = o.pow2_exponent_ceil(x)
        assert 2.0 ** e >= x > 2.0 ** (e - 1)


def test_division_free_reciprocal_of_e4m3_scales():
    # The first kernel forms inv = fp32(1 / (s * 2^gx)) without a division: for
    # s = (1 + m/8) 2^(e-7) it takes fp32(1 / (1 + m/8)) 2^(7-e-gx), for a
    # subnormal s = m 2^-9 it takes fp32(1/m) 2^(9-gx) -- a power-of-two
    # scaling of one of 15 correctly rounded constants.  Equal to the IEEE
    # quotient for every positive E4M3 value and every tensor-scale exponent
    # the kernel accepts.
    rcp_norm = [np.float32(1.0 / (1.0 + m / 8.0)) for m in range(8)]
    rcp_sub = [np.float32(1.0 / m) if m else np.float32(0.0) for m in range(8)]
    for byte in range(1, 0x7F):
        e, m = byte >> 3, byte & 7
        s = (1.0 + m / 8.0) * 2.0 ** (e - 7) if e else m * 2.0 ** -9
        assert s == o.e4m3_decode(np.array([byte]))[0]
        for gx in range(-40, 31):
            want = np.float32(1.0) / np.float32(s * 2.0 ** gx)      # IEEE float32 division
            got = np.float32(float(rcp_norm[m]) * 2.0 ** (7 - e - gx)) if e else \
                np.float32(float(rcp_sub[m]) * 2.0 ** (9 - gx))
            assert got == want, (byte, gx)
