"""Pins of the oracle's NVFP4 tensor scales and of its smoothed activations.

The pages fix FP8 (E4M3) group scales for NVFP4 (SOTA-314 practice page, "Do
this"; NOTE-257 note page, "Key results") and say nothing about the tensor
scale that places the groups in E4M3's range.  The reading used on both sides:
a power of two g = 2^e, the smallest one for which the largest group scale
amax / (6 g) fits E4M3's largest finite value 448 -- for the weights' residual
at calibration-free full range, for the activations with 4x headroom over the
calibration batch.  These tests fix that reading with exact rational
arithmetic and hand-worked values, never by re-evaluating the oracle's own
formula, so a floor for a ceil, a dropped factor 6 or 448, or a lost headroom
factor fails here.
"""
from fractions import Fraction

import numpy as np
import pytest

from oracle import svdq_oracle as o

F32 = np.float32
TOP = Fraction(6 * 448)          # the largest group scale times E2M1's largest value


def _residual_with_amax(a: float, K=32, N=16, seed=0) -> np.ndarray:
    """A float32 [K, N] residual whose largest magnitude is exactly `a`."""
    rng = np.random.default_rng(seed)
    R = (rng.uniform(-1, 1, (K, N)) * 0.5 * a).astype(F32)
    R[3, 5] = F32(-a)
    assert float(np.max(np.abs(R))) == float(F32(a))
    return R


# ---------------------------------------------------------------- weights

@pytest.mark.parametrize("amax,e", [
    (2688.0, 0),                                   # amax / 2688 = 1 = 2^0
    (float(np.nextafter(F32(2688), F32(1e9))), 1),  # one float32 step above -> next power
    (2687.0, 0),
    (1344.0, -1),                                  # exactly half
    (float(np.nextafter(F32(1344), F32(1e9))), 0),
    (1.0, -11),                                    # 2^-12 < 1/2688 <= 2^-11
    (5376.0, 1),
    (3.0 * 2 ** -40, -49),                         # 3 * 2^-40 / 2688 = (8/7) 2^-50, in (2^-50, 2^-49]
])
def test_weight_tensor_exponent_hand_worked(amax, e):
    assert o.weight_tensor_exponent(_residual_with_amax(amax)) == e


def test_weight_tensor_exponent_is_the_smallest_that_fits_e4m3():
    # Definition, in exact rationals: amax / (6 * 448 * 2^e) <= 1 < amax / (6 * 448 * 2^(e-1))
    rng = np.random.default_rng(1)
    for a in (2.0 ** rng.uniform(-60, 60, 400)).astype(F32):
        e = o.weight_tensor_exponent(_residual_with_amax(float(a), K=16, N=16, seed=int(rng.integers(1 << 30))))
        A = Fraction(float(a))
        assert A <= TOP * Fraction(2) ** e, (a, e)
        assert A > TOP * Fraction(2) ** (e - 1), (a, e)


def test_weight_tensor_scale_puts_the_top_group_scale_in_the_last_binade():
    # With that g the largest group's E4M3 scale lands in [224, 448]: it never
    # saturates, and half of g would push it past 448.
    rng = np.random.default_rng(2)
    for a in (2.0 ** rng.uniform(-30, 30, 60)).astype(F32):
        R = _residual_with_amax(float(a), K=64, N=8)
        q = o.quantize_weights(R, "nvfp4")
        top = float(np.max(q["w_scales"]))
        assert 224.0 <= top <= 448.0, (a, top)
        # exact group scale before E4M3 rounding, with half the tensor scale
        assert Fraction(float(a)) / (6 * Fraction(2) ** (q["g_w_exp"] - 1)) > 448


def test_weight_tensor_exponent_of_zero_residual():
    assert o.weight_tensor_exponent(np.zeros((16, 16), dtype=F32)) == 0


# ---------------------------------------------------------------- activations

@pytest.mark.parametrize("x,inv,e", [
    (672.0, 1.0, 0),          # 4 * 672 = 2688: exactly 2^0
    (673.0, 1.0, 1),
    (336.0, 1.0, -1),
    (1344.0, 0.5, 0),         # the smoothed value is 672
    (1.0, 0.5, -10),          # 4 * 0.5 / 2688 = 1/1344 in (2^-11, 2^-10]
    (-672.0, 1.0, 0),         # magnitude, not value
])
def test_activation_tensor_exponent_hand_worked(x, inv, e):
    K = 16
    Xc = np.zeros((3, K), dtype=F32)
    Xc[1, 7] = F32(x)
    Xc[2, 2] = F32(x) * F32(0.25)                  # a smaller entry elsewhere
    inv_lam = np.ones(K, dtype=F32)
    inv_lam[7] = F32(inv)
    assert o.activation_tensor_exponent(Xc, inv_lam) == e


def test_activation_tensor_exponent_keeps_4x_headroom():
    # exact rationals: 4 amax / (6 * 448 * 2^e) <= 1 < 4 amax / (6 * 448 * 2^(e-1)),
    # i.e. the calibration batch's largest group scale amax / (6 * 2^e) lies
    # in (56, 112]: four times below E4M3's 448
    rng = np.random.default_rng(3)
    for a in (2.0 ** rng.uniform(-40, 40, 300)).astype(F32):
        Xc = np.zeros((2, 64), dtype=F32)
        Xc[1, 9] = a
        e = o.activation_tensor_exponent(Xc, np.ones(64, dtype=F32))
        top = Fraction(float(a)) / (6 * Fraction(2) ** e)
        assert Fraction(56) < top <= Fraction(112), (a, e, float(top))


def test_activation_tensor_exponent_uses_smoothed_values():
    # the largest raw entry is not the largest smoothed one
    Xc = np.array([[1000.0, 10.0]], dtype=F32)
    inv_lam = np.array([0.001, 100.0], dtype=F32)      # smoothed: ~1.0 and 1000
    e = o.activation_tensor_exponent(Xc, inv_lam)
    v = Fraction(float(F32(F32(10.0) * F32(100.0))))
    assert 4 * v <= TOP * Fraction(2) ** e and 4 * v > TOP * Fraction(2) ** (e - 1)


# ---------------------------------------------------------------- smoothed activations

def test_smoothed_activations_one_float32_multiply():
    # x * fp32(1/3) for x = 3 is exactly 1 + 2^-25 in real arithmetic; a single
    # float32 rounding gives 1.0 (a float64 product would keep the 2^-25)
    inv = np.array([F32(1.0 / 3.0), F32(1.0 / 7.0), F32(0.7)], dtype=F32)
    X = np.array([[3.0, 7.0, 3.0]], dtype=F32)
    got = o.smoothed_activations(X, inv)
    assert got.dtype == np.float32
    assert Fraction(float(inv[0])) * 3 == 1 + Fraction(1, 2 ** 25)
    assert got[0, 0] == F32(1.0)
    assert got[0, 1] == F32(1.0)                        # 7 * fp32(1/7) = 1 + 3 * 2^-26
    assert got[0, 2].view(np.uint32) == 0x40066666      # float32(2.1): 3 * fp32(0.7) rounds down to it
    # a product that needs no rounding passes through unchanged
    assert o.smoothed_activations(np.array([[1.5]], dtype=F32), np.array([0.25], dtype=F32))[0, 0] == F32(0.375)
