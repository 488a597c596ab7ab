"""Pins of the oracle's W8A8 variant (rank 16 at 8 bits; SOTA-314 practice
page, "Do this"; NOTE-257 note page, "Key results").  The pages give no 8-bit
group size; the oracle reads one group per row -- per token for activations,
per output channel for the residual -- with float32 scales.

Pinned by: hand-worked rows whose scale is a power of two (codes are then the
ties-to-even rounding of v / s, written out), the per-element round-trip bound
s/2, the row maximum landing on +-127, zero rows, and an exact rational brute
force of the layer output from decoded codes and scales.
"""
from fractions import Fraction

import numpy as np
import pytest

import synthetic as syn
from oracle import svdq_oracle as o

F32 = np.float32


def test_scale_of_127_is_exactly_one_and_codes_round_half_even():
    v = np.array([[127.0, -63.5, 2.5, -0.5, 3.49, 0.0, -126.6, 64.5]], dtype=F32)
    q = o.int8_quantize_rows(v)
    assert q["scales"][0] == 1.0                  # fp32(127 * fp32(1/127)) rounds to exactly 1
    np.testing.assert_array_equal(q["codes"][0], [127, -64, 2, 0, 3, 0, -127, 64])


@pytest.mark.parametrize("k", [-20, -3, 4, 40])
def test_power_of_two_scales(k):
    # a = 127 2^k: s = 2^k exactly, so code = rint_even(v / 2^k)
    rng = np.random.default_rng(k + 100)
    v = (rng.integers(-254, 255, size=(3, 64)) / 2.0).astype(F32)          # multiples of 1/2, ties included
    v[:, 0] = 127.0
    v = (v * F32(2.0 ** k)).astype(F32)
    q = o.int8_quantize_rows(v)
    np.testing.assert_array_equal(q["scales"], np.full(3, 2.0 ** k))
    want = np.clip(np.rint(v.astype(np.float64) / 2.0 ** k), -127, 127)
    np.testing.assert_array_equal(q["codes"], want.astype(np.int8))


def test_round_trip_bound_row_max_and_zero_rows():
    rng = np.random.default_rng(7)
    v = (rng.standard_normal((50, 96)) * rng.uniform(1e-3, 1e3, size=(50, 1))).astype(F32)
    v[3] = 0.0
    q = o.int8_quantize_rows(v)
    s = q["scales"]
    assert s[3] == 0 and np.all(q["codes"][3] == 0)
    err = np.abs(q["deq"] - v.astype(np.float64))
    assert np.all(err <= s[:, None] * (0.5 + 1e-6))
    live = np.arange(50) != 3
    assert np.all(np.max(np.abs(q["codes"][live].astype(int)), axis=1) == 127)


def test_forward_exact_rational_brute_force():
    d = syn.custom_layer(301, M=3, K=64, N=16)
    p = o.prepare(d["W"], d["bias"], d["Xc"], fmt="w8a8", rank=16)
    assert p["rank"] == 16
    xq = o.quantize_activations(d["X"], p["inv_lam"], "w8a8")
    XL = o.down_projection(d["X"], p["L1d"])
    y = o.forward(p, d["X"])["Y"]
    for m in range(3):
        for n in range(16):
            acc = sum(Fraction(int(xq["codes"][m, k])) * Fraction(int(p["w_codes"][n, k])) for k in range(64))
            v = acc * Fraction(float(xq["scales"][m])) * Fraction(float(p["w_scales"][n]))
            v += sum(Fraction(float(XL[m, i])) * Fraction(float(p["L2b"][i, n])) for i in range(16))
            v += Fraction(float(p["bias"][n]))
            assert abs(float(v) - y[m, n]) <= 1e-12 * max(1.0, abs(float(v)))


def test_eight_bits_track_the_layer_better_than_four():
    d = syn.custom_layer(302, M=128, K=512, N=256)
    exact = d["X"].astype(np.float64) @ d["W"] + d["bias"]
    e8 = np.linalg.norm(o.forward(o.prepare(d["W"], d["bias"], d["Xc"], fmt="w8a8", rank=16), d["X"])["Y"] - exact)
    e4 = np.linalg.norm(o.forward(o.prepare(d["W"], d["bias"], d["Xc"], fmt="nvfp4", rank=32), d["X"])["Y"] - exact)
    assert e8 < 0.5 * e4
