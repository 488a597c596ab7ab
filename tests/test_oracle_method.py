"""Pins of the oracle's method steps (smoothing, SVD split, residual, forward,
ablation) against closed forms, planted spectra, exact rational brute force,
special cases and the inequalities the pages state.

Sources: SOTA-314 practice page ("Do this"); NOTE-257 note page ("Key
results": Propositions 4.1/4.2, Eckart-Young, Figure 5, the LoRC control;
"Claims" C1 and C3).
"""
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

import synthetic as syn
from oracle import svdq_oracle as o

F32 = np.float32


# ---------------------------------------------------------------- smoothing

def test_smoothing_hand_worked():
    Xc = np.array([[4.0, -1.0, 0.0], [-2.0, 9.0, 0.0]], dtype=F32)
    W = np.array([[0.25, -0.5], [1.0, 4.0], [3.0, 0.0]], dtype=F32)
    lam, inv = o.smoothing_factors(Xc, W, 0.5)
    # ax = (4, 9, 0), aw = (0.5, 4, 3): lam = (sqrt(4)/sqrt(0.5), 3/2, 1 (ax = 0))
    assert lam[1] == 1.5 and lam[2] == 1.0 and inv[1] == F32(1 / 1.5)
    assert abs(float(lam[0]) - 2 * np.sqrt(2)) <= np.spacing(F32(2.8284271))


def test_smoothing_alpha_closed_forms():
    rng = np.random.default_rng(5)
    Xc = rng.standard_normal((16, 8)).astype(F32)
    W = rng.standard_normal((8, 4)).astype(F32)
    ax = np.max(np.abs(Xc), axis=0)
    aw = np.max(np.abs(W), axis=1)
    lam1, _ = o.smoothing_factors(Xc, W, 1.0)       # lam = max|X|
    lam0, _ = o.smoothing_factors(Xc, W, 0.0)       # lam = 1 / max|W|
    np.testing.assert_array_equal(lam1, ax)
    np.testing.assert_allclose(lam0, 1.0 / aw, rtol=2 ** -23)
    # the alpha = 0.5 float32 path agrees with the general float64 path to 1 ulp
    lam_h, _ = o.smoothing_factors(Xc, W, 0.5)
    lam_g = o.fp32(np.sqrt(ax.astype(np.float64) / aw.astype(np.float64)))
    assert np.all(np.abs(lam_h - lam_g) <= np.spacing(lam_g))


def test_smoothing_equalizes_channel_ranges():
    # after smoothing, max|X^|_k = max|W^|_k = sqrt(ax aw): the outlier moves into W
    d = syn.layer("tiny")
    lam, inv = o.smoothing_factors(d["Xc"], d["W"])
    ax = np.max(np.abs(d["Xc"]), axis=0).astype(np.float64)
    aw = np.max(np.abs(d["W"]), axis=1).astype(np.float64)
    np.testing.assert_allclose(ax / lam, np.sqrt(ax * aw), rtol=1e-6)
    np.testing.assert_allclose(aw * lam, np.sqrt(ax * aw), rtol=1e-6)


def test_smoothing_preserves_product():
    d = syn.layer("tiny")
    lam, inv = o.smoothing_factors(d["Xc"], d["W"])
    X = d["X"].astype(np.float64)
    lhs = (X * inv.astype(np.float64)) @ (lam.astype(np.float64)[:, None] * d["W"])
    rhs = X @ d["W"]
    assert np.linalg.norm(lhs - rhs) <= 1e-6 * np.linalg.norm(rhs)


# ---------------------------------------------------------------- SVD split

def _planted(K, N, n, seed):
    rng = np.random.default_rng(seed)
    A, _ = np.linalg.qr(rng.standard_normal((K, n)))
    B, _ = np.linalg.qr(rng.standard_normal((N, n)))
    s = np.sort(rng.uniform(0.1, 10, n))[::-1] * np.linspace(3, 1, n)
    return A, s, B


def test_svd_split_recovers_planted_top_r():
    A, s, B = _planted(96, 64, 48, 7)
    W = (A * s) @ B.T
    r = 8
    L1, L2, S = o.svd_split(W, r)
    assert L1.shape == (96, r) and L2.shape == (r, 64)
    np.testing.assert_allclose(L1 @ L2, (A[:, :r] * s[:r]) @ B[:, :r].T, atol=1e-10)
    # Eckart-Young: the truncation error is the planted tail
    np.testing.assert_allclose(np.linalg.norm(W - L1 @ L2) ** 2, np.sum(s[r:] ** 2), rtol=1e-10)
    # L2 rows are orthonormal; L1 columns are orthogonal with norms sigma_i
    np.testing.assert_allclose(L2 @ L2.T, np.eye(r), atol=1e-12)
    np.testing.assert_allclose(np.linalg.norm(L1, axis=0), s[:r], rtol=1e-12)


def test_eckart_young_on_smoothed_synthetic_weight():
    # tail energy against the eigenvalues of W^T W (a symmetric eigensolver,
    # not the SVD routine the oracle calls)
    d = syn.layer("tiny")
    p = o.prepare(d["W"], d["bias"], d["Xc"])
    W_hat = p["lam"].astype(np.float64)[:, None] * d["W"]
    ev = np.sort(np.linalg.eigvalsh(W_hat.T @ W_hat))[::-1]
    tail = np.sum(np.clip(ev[32:], 0, None))
    np.testing.assert_allclose(np.linalg.norm(W_hat - p["L1"] @ p["L2"]) ** 2, tail, rtol=1e-6)


def test_residual_is_smoothed_weight_minus_stored_branch():
    d = syn.layer("tiny")
    p = o.prepare(d["W"], d["bias"], d["Xc"])
    W_hat = p["lam"].astype(np.float64)[:, None] * d["W"]
    exact_res = W_hat - p["L1"] @ p["L2"]
    rounding = np.linalg.norm(p["lam"].astype(np.float64)[:, None] * p["L1d"] @ p["L2b"] - p["L1"] @ p["L2"])
    fp32_err = np.linalg.norm(p["R"]) * 2 ** -24 * 4
    assert np.linalg.norm(p["R"] - exact_res) <= rounding + fp32_err
    # the stored branch is BF16 (L1d carries 1/lam)
    np.testing.assert_array_equal(o.bf16_round(p["L1d"]), p["L1d"])
    np.testing.assert_array_equal(o.bf16_round(p["L2b"]), p["L2b"])
    np.testing.assert_allclose(p["L1d"] * p["lam"][:, None], p["L1"], rtol=2 ** -7, atol=1e-30)


def test_steep_spectrum_rank32_removes_magnitude():
    # Figure 5 premise on the synthetic stand-in: rank 32 of W_hat carries a
    # large share of its energy, and the residual fed to the quantizer is smaller.
    d = syn.layer("tiny")
    p = o.prepare(d["W"], d["bias"], d["Xc"])
    W_hat = p["lam"].astype(np.float64)[:, None] * d["W"]
    assert np.linalg.norm(p["R"]) < 0.7 * np.linalg.norm(W_hat)


# ---------------------------------------------------------------- forward

def _exact_forward(p, X, fmt):
    """Exact rational evaluation from the stored codes and scales, decoded from
    their bit fields (independent of the oracle's float64 matmul)."""
    def e2m1(c):
        s, e, m = (c >> 3) & 1, (c >> 1) & 3, c & 1
        v = Fraction(m, 2) if e == 0 else (1 + Fraction(m, 2)) * Fraction(2) ** (e - 1)
        return -v if s else v

    def e4m3(b):
        e, m = (b >> 3) & 0xF, b & 7
        return Fraction(m, 8) * Fraction(2) ** -6 if e == 0 else (1 + Fraction(m, 8)) * Fraction(2) ** (e - 7)

    xq = o.quantize_activations(X, p["inv_lam"], fmt, p["g_x_exp"])
    M, K = X.shape
    N = p["N"]
    if fmt == "nvfp4":
        gx, gw = Fraction(2) ** p["g_x_exp"], Fraction(2) ** p["g_w_exp"]
        dx = [[e2m1(int(xq["codes"][m, k])) * e4m3(int(xq["scale_bytes"][m, k // 16])) * gx
               for k in range(K)] for m in range(M)]
        dw = [[e2m1(int(p["w_codes"][n, k])) * e4m3(int(p["w_scale_bytes"][n, k // 16])) * gw
               for k in range(K)] for n in range(N)]
    else:
        dx = [[Fraction(int(xq["codes"][m, k])) * Fraction(float(xq["scales"][m, k // 64]))
               for k in range(K)] for m in range(M)]
        dw = [[Fraction(int(p["w_codes"][n, k])) * Fraction(float(p["w_scales"][n, k // 64]))
               for k in range(K)] for n in range(N)]
    XL = [[sum(Fraction(float(X[m, k])) * Fraction(float(p["L1d"][k, j])) for k in range(K))
           for j in range(p["rank"])] for m in range(M)]
    Y = np.empty((M, N))
    for m in range(M):
        xl = [Fraction(float(o.bf16_round(float(v)))) for v in XL[m]]
        for n in range(N):
            acc = sum(dx[m][k] * dw[n][k] for k in range(K))
            acc += sum(xl[j] * Fraction(float(p["L2b"][j, n])) for j in range(p["rank"]))
            acc += Fraction(float(p["bias"][n]))
            Y[m, n] = float(acc)
    return Y


@pytest.mark.parametrize("fmt,K,rank", [("nvfp4", 16, 4), ("nvfp4", 32, 8), ("nvfp4", 64, 8), ("int4", 64, 4)])
def test_forward_equals_exact_rational(fmt, K, rank):
    d = syn.custom_layer(seed=K + rank, M=6, K=K, N=12, sigma0=5.0, calib_tokens=16)
    p = o.prepare(d["W"], d["bias"], d["Xc"], fmt=fmt, rank=rank)
    got = o.forward(p, d["X"])["Y"]
    want = _exact_forward(p, d["X"], fmt)
    np.testing.assert_allclose(got, want, rtol=2 ** -50, atol=2 ** -60)


def test_zero_input_gives_bias():
    d = syn.layer("tiny")
    p = o.prepare(d["W"], d["bias"], d["Xc"])
    f = o.forward(p, np.zeros((4, 512), dtype=F32))
    np.testing.assert_array_equal(f["Y_bf16"], np.broadcast_to(o.bf16_round(d["bias"]), (4, 512)))


def test_rank_zero_is_plain_w4a4():
    d = syn.layer("tiny")
    p = o.prepare(d["W"], d["bias"], d["Xc"], rank=0)
    lam = p["lam"].astype(np.float64)
    np.testing.assert_array_equal(p["R"], o.fp32(lam[:, None] * d["W"]))
    xq = o.quantize_activations(d["X"], p["inv_lam"], "nvfp4", p["g_x_exp"])
    want = xq["deq"] @ p["w_deq"].T + d["bias"]
    np.testing.assert_array_equal(o.forward(p, d["X"])["Y"], want)


def test_gelu_tanh_matches_torch():
    y = np.linspace(-8, 8, 2001)
    want = torch.nn.functional.gelu(torch.from_numpy(y), approximate="tanh").numpy()
    np.testing.assert_allclose(o.gelu_tanh(y), want, rtol=1e-14, atol=1e-15)


def test_gelu_tanh_tail_against_300_digit_tanh_form():
    # the tanh form 0.5 y (1 + tanh(u)) evaluated with 300 significant digits
    # (decimal arithmetic, tanh from exp) keeps its relative accuracy where
    # float64's 1 + tanh(u) cancels: the oracle must match it all the way down
    # the negative tail, to 1e-12 relative (float64's exp(-2u) carries the
    # rounding of u amplified by |2u| <= 300)
    from decimal import Decimal, getcontext
    getcontext().prec = 300
    k0 = (Decimal(2) / Decimal(str(math.pi))).sqrt()

    def ref(v):
        y = Decimal(float(v))
        u = k0 * (y + Decimal("0.044715") * y ** 3)
        e = (2 * u).exp()
        return float(Decimal("0.5") * y * (1 + (e - 1) / (e + 1)))

    ys = np.array([-12.0, -10.0, -9.5, -8.0, -6.0, -5.0, -3.0, -1.0, -0.25, 0.0, 0.5, 2.0, 7.0])
    got = o.gelu_tanh(ys)
    want = np.array([ref(v) for v in ys])
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=0.0)
    assert got[0] < 0 and abs(got[0]) > 1e-70               # about -1.6e-61: not flushed to zero


# ---------------------------------------------------------------- theory and ablation

def test_proposition_4_1_textbook_bound():
    # ||XW - Q(X)Q(W)|| <= ||X|| ||W - Q(W)|| + ||X - Q(X)|| (||W|| + ||W - Q(W)||)
    d = syn.layer("tiny")
    X, W = d["X"].astype(np.float64), d["W"].astype(np.float64)
    qx = o._qx(d["X"], "nvfp4", d["Xc"])
    qw = o._qw(d["W"], "nvfp4")
    lhs = np.linalg.norm(X @ W - qx @ qw)
    ew, ex = np.linalg.norm(W - qw), np.linalg.norm(X - qx)
    rhs = np.linalg.norm(X) * ew + ex * (np.linalg.norm(W) + ew)
    assert lhs <= rhs


def test_ablation_ordering_tiny():
    # decompose-then-quantize beats LoRC (C1), smoothing on top helps further
    d = syn.layer("tiny", with_heldout=True)
    e = o.ablation_errors(d["W"], d["bias"], d["Xc"], d["Xh"])
    assert e["dtq"] < e["lorc"]
    assert e["svdquant"] < e["lorc_smooth"]
    assert e["svdquant"] < e["dtq"]
    assert e["svdquant"] < e["smooth"] < e["naive"]


def test_quantization_error_spectrum_is_flat():
    # C3 (diagnostic): W - Q(W) has a well-spread spectrum, W a steep one
    d = syn.layer("tiny")
    W = d["W"].astype(np.float64)
    E = W - o._qw(d["W"], "nvfp4")
    sw = np.linalg.svd(W, compute_uv=False)
    se = np.linalg.svd(E, compute_uv=False)
    assert sw[0] / np.median(sw) > 10
    assert se[0] / np.median(se) < 5


def test_w4a16_forward():
    rng = np.random.default_rng(9)
    W = syn.to_bf16(rng.standard_normal((128, 64)) / 8)
    X = syn.to_bf16(rng.standard_normal((4, 128)))
    b = syn.to_bf16(rng.standard_normal(64) * 0.1)
    p = o.w4a16_prepare(W, b)
    f = o.w4a16_forward(p, X)
    np.testing.assert_allclose(f["Y"], X.astype(np.float64) @ p["w_deq"].T + b, rtol=1e-13)
    s = np.repeat(p["w_scales"], 64, axis=1)
    assert np.all(np.abs(W.T - p["w_deq"]) <= s / 2 * (1 + 1e-6))


def test_svd_split_rank_above_matrix_rank_pads_zeros():
    # r larger than min(K, N): the branch carries the whole matrix, the residual is zero
    rng = np.random.default_rng(8)
    W = rng.standard_normal((64, 16))
    L1, L2, S = o.svd_split(W, 32)
    assert L1.shape == (64, 32) and L2.shape == (32, 16)
    assert np.all(L1[:, 16:] == 0) and np.all(L2[16:] == 0)
    np.testing.assert_allclose(L1 @ L2, W, atol=1e-12)
