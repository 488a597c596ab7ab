"""Pins of the oracle's group quantizers: hand-worked groups, zero and tiny
groups, saturation, and the per-element round-trip bound that Proposition 4.2
rests on (a matrix's rounding error is bounded by its own magnitude; NOTE-257
note page, "Key results").
"""
import numpy as np
import pytest

from oracle import svdq_oracle as o

F32 = np.float32


def test_nvfp4_hand_worked_group_scale_one():
    # a = 6, g = 1: t = fp32(6 * fp32(1/6)) = 1.0 -> s = E4M3(1.0) = 0x38, inv = 1, q = v.
    v = np.array([[6.0, 3.0, 1.5, 0.75, -0.75, 0.3, 0.0, -6.0,
                   2.9, 5.5, 0.1, 1.0, -1.0, 4.0, 0.25, -0.2]], dtype=F32)
    q = o.nvfp4_quantize(v, 0)
    assert q["scale_bytes"][0, 0] == 0x38 and q["scales"][0, 0] == 1.0
    assert list(q["codes"][0]) == [7, 5, 3, 2, 10, 1, 0, 15, 5, 7, 0, 2, 10, 6, 0, 8]


def test_nvfp4_hand_worked_group_rounded_scale():
    # a = 10, g = 2^-3: c = fp32(1/6) * 8, t = fp32(10 c) = 13.333334 -> E4M3 13.0
    # (binade [8,16), quantum 1) = byte 0b0_1010_101 = 0x55; s*g = 1.625,
    # inv = fp32(1/1.625) = 0.61538464; q(10) = 6.15 -> 6 (code 7),
    # q(5) = 3.08 -> 3 (code 5), q(4) = 2.46 -> 2 (code 4), q(-1) = -0.615 -> -0.5 (code 9).
    v = np.zeros((1, 16), dtype=F32)
    v[0, :4] = [10.0, 5.0, 4.0, -1.0]
    q = o.nvfp4_quantize(v, -3)
    assert q["scale_bytes"][0, 0] == 0x55
    assert q["scales"][0, 0] * 2.0 ** -3 == 1.625
    assert list(q["codes"][0, :4]) == [7, 5, 4, 9]
    assert np.all(q["codes"][0, 4:] == 0)


def test_nvfp4_zero_tiny_and_signed_zero():
    v = np.zeros((3, 16), dtype=F32)
    v[1, :] = 1e-8                         # t rounds below half the smallest subnormal scale
    v[2, 0] = 6.0
    v[2, 1] = -0.01                        # rounds to -0: code 0b1000
    q = o.nvfp4_quantize(v, 0)
    assert np.all(q["codes"][0] == 0) and q["scale_bytes"][0, 0] == 0
    assert np.all(q["codes"][1] == 0) and q["scale_bytes"][1, 0] == 0
    assert q["codes"][2, 1] == 8


def test_nvfp4_subnormal_scale():
    # a = 0.006, g = 1: t = 0.001 -> nearest E4M3 subnormal is 2^-9 (byte 0x01)
    v = np.zeros((1, 16), dtype=F32)
    v[0, 0] = 0.006
    q = o.nvfp4_quantize(v, 0)
    assert q["scale_bytes"][0, 0] == 0x01
    # q = fp32(0.006 * fp32(1 / 2^-9)) = 3.07 -> 3.0, code 5
    assert q["codes"][0, 0] == 5


def test_nvfp4_scale_saturation():
    # t > 448 saturates the scale at 448; codes saturate at +-6
    v = np.zeros((1, 16), dtype=F32)
    v[0, 0] = 6000.0
    v[0, 1] = -3000.0
    q = o.nvfp4_quantize(v, 0)
    assert q["scale_bytes"][0, 0] == 0x7E
    assert q["codes"][0, 0] == 7 and q["codes"][0, 1] == 15


def _halfstep(qabs):
    return np.where(qabs <= 2, 0.25, np.where(qabs <= 4, 0.5, 1.0))


@pytest.mark.parametrize("scale_pow,headroom", [(-8, 0), (-2, 2), (0, 0), (3, 5)])
def test_nvfp4_round_trip_bound(scale_pow, headroom):
    rng = np.random.default_rng(100 + scale_pow)
    v = (rng.standard_normal((64, 256)) * 2.0 ** scale_pow
         * 10.0 ** rng.uniform(-4, 1, (64, 1))).astype(F32)
    v[:, :16] *= 30
    # tensor scale from the data (as the method picks it), plus optional headroom
    g_exp = o.pow2_exponent_ceil(float(np.max(np.abs(v))) / (6 * 448)) + headroom
    q = o.nvfp4_quantize(v, g_exp)
    s = np.repeat(q["scales"], 16, axis=1) * 2.0 ** g_exp
    a = np.repeat(np.max(np.abs(v.reshape(64, 16, 16)), axis=2), 16, axis=1)
    err = np.abs(v.astype(np.float64) - q["deq"])
    nz = s > 0
    qabs = np.abs(v.astype(np.float64)) / np.where(nz, s, 1)
    # |q| <= 6: half the local E2M1 step times the group scale.  |q| > 6 means
    # the code saturated: with a normal E4M3 scale (relative rounding <= 2^-4)
    # q <= 6 (1 + 2^-4), so the error stays below 0.375 s g; with a subnormal
    # scale (absolute rounding <= 2^-10 before the tensor scale g) the error
    # is at most 6 * 2^-10 * g.
    g = 2.0 ** g_exp
    normal = np.repeat(q["scales"], 16, axis=1) >= 2.0 ** -6
    sat_bound = np.where(normal, 0.375 * s, 6 * 2.0 ** -10 * g)
    bound = np.where(qabs <= 6, _halfstep(qabs) * s, sat_bound) * (1 + 1e-6)
    assert np.all(err[nz] <= bound[nz])
    assert np.all(err[~nz] <= a[~nz])
    if headroom >= 5:
        assert np.any(nz & ~normal)         # the subnormal-scale branch is exercised
    # zero-scale groups only when a < 6 * g * 2^-10 (half the smallest subnormal scale)
    assert np.all(a[~nz] < 6 * 2.0 ** g_exp * 2.0 ** -10 * (1 + 1e-6))
    if headroom >= 5:
        assert np.any(~nz)                  # the tiny-group branch is exercised


def test_int4_hand_worked_group():
    # a = 7: s = bf16(fp32(7 * fp32(1/7))) = 1.0, inv = 1: codes = rint_even(v)
    v = np.zeros((1, 64), dtype=F32)
    v[0, :7] = [7.0, -7.0, 3.5, 2.5, 1.49, -0.5, 0.6]
    q = o.int4_quantize(v)
    assert q["scales"][0, 0] == 1.0
    assert list(q["codes"][0, :7]) == [7, -7, 4, 2, 1, 0, 1]


def test_int4_scale_is_bf16_of_a_over_7():
    v = np.zeros((1, 64), dtype=F32)
    v[0, 0] = 1.0
    q = o.int4_quantize(v)
    # fp32(1/7) = 0.142857149 -> bf16 keeps 8 significant bits: 0.142578125 (= 73/512)
    assert q["scales"][0, 0] == 73 / 512
    # q = fp32(1 / 0.142578125) = 7.0137 -> clamps to 7
    assert q["codes"][0, 0] == 7


def test_int4_round_trip_bound():
    rng = np.random.default_rng(20)
    v = (rng.standard_normal((32, 512)) * 10.0 ** rng.uniform(-3, 2, (32, 1))).astype(F32)
    q = o.int4_quantize(v)
    s = np.repeat(q["scales"], 64, axis=1)
    err = np.abs(v.astype(np.float64) - q["deq"])
    assert np.all(err <= s / 2 * (1 + 1e-6))
    assert np.all(np.abs(q["codes"]) <= 7)
