"""The INT4 GEMM multiplies FP16 operands c * h, where c is an INT4 code in
[-7, 7] and h = fp16(s * 2^-e) is the group's BF16 scale s moved by ONE
power-of-two range exponent e per layer and operand (the weights' e from their
largest residual magnitude, the activations' e from the calibration batch),
and relies on both h and c * h being exact in FP16.

c needs 3 significant bits and s 8, so c * s has at most 11 -- FP16's
precision.  Exactness then only needs the value to stay within FP16's range:
  * at the top, the kernel clamps h at 8192 (7 * 8192 < 65504, FP16's largest);
  * at the bottom, FP16 subnormals are multiples of 2^-24, so every BF16 scale
    with s * 2^-e >= 2^-17 (8 significant bits, the lowest at 2^-24) is exact;
    a smaller scale is rounded to a multiple of 2^-24 (error at most 2^-25 in
    units of 2^e).
Checked here for every code and every BF16 scale of the window, for several
range exponents, and the window is placed against the kernel's rules for e.
"""
import math

import numpy as np
import pytest

CLAMP = 8192.0          # the activation clamp of the INT4 GEMM (FP16 operand units)
LOW = 2.0 ** -17        # the smallest BF16 scale (in operand units) that is always exact


def _bf16_values():
    bits = np.arange(1 << 16, dtype=np.uint32)
    with np.errstate(invalid="ignore"):              # the NaN patterns, dropped below
        v = (bits << 16).view(np.float32).astype(np.float64)
    return v[np.isfinite(v) & (v > 0)]


def _exact_in_fp16(v: np.ndarray) -> bool:
    with np.errstate(over="ignore"):
        return bool(np.array_equal(v.astype(np.float16).astype(np.float64), v))


@pytest.mark.parametrize("e", [-30, -5, 0, 7, 40])
def test_every_code_times_every_bf16_scale_in_the_window_is_exact(e):
    s = _bf16_values()
    h_exact = s * 2.0 ** -e                         # exact: power-of-two scaling in float64
    win = (h_exact >= LOW) & (h_exact <= CLAMP)
    h = h_exact[win]
    assert h.size == 30 * 128 + 1                   # 30 binades of 128 BF16 values, and 8192 itself
    assert _exact_in_fp16(h)                        # the FP16 scale itself
    h16 = h.astype(np.float16)
    for c in range(-7, 8):
        prod = (np.float16(c) * h16).astype(np.float64)   # FP16 multiply (__hmul2), correctly rounded
        assert np.array_equal(prod, c * h), c


def test_below_the_window_values_round_to_multiples_of_2_pow_minus_24():
    s = _bf16_values()
    h = s[(s < LOW) & (s >= 2.0 ** -30)]
    assert not _exact_in_fp16(h)                    # some do lose bits below the window
    r = h.astype(np.float16).astype(np.float64)
    assert np.all(np.abs(r - h) <= 2.0 ** -25)
    assert np.all(np.mod(r, 2.0 ** -24) == 0)


def test_a_scale_with_more_bits_would_not_be_exact():
    # the bound is tight: 511/256 has a 9-bit significand (not a BF16 value),
    # and 7 * 511 = 3577 needs 12 bits
    s = 511.0 / 256.0
    assert float(np.float16(7 * s)) != 7 * s


def _ceil_log2(x: float) -> int:
    m, e = math.frexp(x)
    return e - 1 if m == 0.5 else e


@pytest.mark.parametrize("x_amax", [1e-3, 0.37, 1.0, 50.0, 3072.0, 6.5e4])
def test_activation_exponent_window_covers_calibration_range_with_headroom(x_amax):
    # The layer fixes e_x = ceil(log2(amax of the smoothed calibration batch)) - 8.
    # A calibration group scale is at most amax / 7 (times BF16 rounding), a
    # runtime group 220x larger still stays below the clamp, and every group
    # scale down to 2^-24 of amax stays exact.
    ex = _ceil_log2(x_amax) - 8
    top_calib = x_amax / 7.0 * (1 + 2.0 ** -8)
    assert 220 * top_calib * 2.0 ** -ex <= CLAMP
    assert x_amax * 2.0 ** -24 * 2.0 ** -ex >= LOW


@pytest.mark.parametrize("r_amax", [1e-4, 0.02, 1.0, 9.0, 700.0])
def test_weight_exponent_window_covers_all_residual_groups(r_amax):
    # The layer fixes e_w = ceil(log2(amax |R|)) - 14: the largest |c h| is at
    # most 2^14 (below FP16's 65504) and every scale down to 2^-30 of amax is exact.
    ew = _ceil_log2(r_amax) - 14
    s_top = r_amax / 7.0 * (1 + 2.0 ** -8)
    assert 7 * s_top * 2.0 ** -ew <= 2.0 ** 14 * (1 + 2.0 ** -8) < 65504
    assert r_amax * 2.0 ** -30 * 2.0 ** -ew >= LOW
