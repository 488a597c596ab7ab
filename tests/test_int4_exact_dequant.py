"""The INT4 GEMM multiplies FP16 operands c * s * 2^-e (c an INT4 code in
[-7, 7], s a BF16 group scale, e a power-of-two range exponent) and relies on
each being exact in FP16: c needs 3 significant bits and s 8, so c * s has at
most 11 -- FP16's precision -- as long as it stays in FP16's normal range.
Checked here for every positive finite BF16 scale and every code, with the
range exponent placing the scale below the kernel's clamp of 8192."""
import numpy as np


def _bf16_values():
    bits = np.arange(1 << 16, dtype=np.uint32)
    with np.errstate(invalid="ignore"):              # the NaN patterns, dropped below
        v = (bits << 16).view(np.float32).astype(np.float64)
    return v[np.isfinite(v) & (v > 0)]


def test_every_code_times_every_bf16_scale_is_exact_in_fp16():
    s = _bf16_values()
    # the range exponent: scale the largest value of each binade into [2^11, 2^12)
    # (any power of two that keeps c * s within FP16's normal range will do)
    e = np.floor(np.log2(s))
    shifted = s * np.exp2(11 - e)                  # exact: power-of-two scaling in float64
    assert np.all(shifted < 8192)                  # below the kernel's clamp
    for c in range(-7, 8):
        v = c * shifted                            # exact in float64
        h = v.astype(np.float16).astype(np.float64)
        assert np.array_equal(h, v), c


def test_a_scale_with_more_bits_would_not_be_exact():
    # the bound is tight: 511/256 has a 9-bit significand (not a BF16 value),
    # and 7 * 511 = 3577 needs 12 bits
    s = 511.0 / 256.0
    assert float(np.float16(7 * s)) != 7 * s
