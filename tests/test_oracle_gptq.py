"""Pins of the oracle's GPTQ residual quantizer.

The SOTA-314 practice page ("Do this") quantizes the residual with GPTQ rather
than round-to-nearest; the NOTE-257 note page ("Key results") reports the
quality with it.  The pages do not restate GPTQ, so the oracle follows the
published algorithm (Frantar et al. 2022).  These tests pin it to things other
than itself:

* a hand-worked damped Hessian (dead channel, 1% damping);
* the Cholesky factor against its defining property;
* a diagonal Hessian, where the error feedback vanishes and GPTQ is exactly
  round-to-nearest;
* a brute-force Optimal Brain Surgeon pass that recomputes the inverse of the
  remaining-coordinates Hessian at every step (no Cholesky at all) and must
  feed the quantizer the same values and reach the same codes;
* the claim itself: lower calibration-output error than round-to-nearest on
  correlated activations, and on a held-out batch.
"""
import numpy as np
import pytest

import synthetic as syn
from oracle import svdq_oracle as o

F32 = np.float32


def test_hessian_hand_worked():
    # X_hat = Xc (inv_lam = 1): H = [[1+4, 0], [0, 0]]; the dead channel gets 1,
    # then 1% of the mean diagonal (5 + 1) / 2 = 3 is added: 0.03
    Xc = np.array([[1.0, 0.0], [2.0, 0.0]], dtype=F32)
    H = o.gptq_hessian(Xc, np.ones(2, dtype=F32))
    np.testing.assert_allclose(H, [[5.03, 0.0], [0.0, 1.03]], rtol=0, atol=1e-15)
    # the smoothing enters: inv_lam = (0.5, 1) halves channel 0 before the product
    Xc2 = np.array([[2.0, 1.0], [0.0, 3.0]], dtype=F32)
    H2 = o.gptq_hessian(Xc2, np.array([0.5, 1.0], dtype=F32), damp=0.0)
    np.testing.assert_array_equal(H2, [[1.0, 1.0], [1.0, 10.0]])


def test_factor_definition():
    rng = np.random.default_rng(3)
    X = rng.standard_normal((40, 24))
    H = X.T @ X + 0.1 * np.eye(24)
    U = o.gptq_factor(H)
    assert np.all(np.tril(U, -1) == 0) and np.all(np.diag(U) > 0)
    np.testing.assert_allclose(U.T @ U @ H, np.eye(24), atol=1e-10)


def _orthogonal_calibration(K):
    # one nonzero per row and column: X_hat^T X_hat is diagonal
    rng = np.random.default_rng(11)
    return np.diag(syn.to_bf16(rng.uniform(0.5, 4.0, K))).astype(F32)


@pytest.mark.parametrize("fmt", ["nvfp4", "int4"])
def test_diagonal_hessian_reduces_to_rtn(fmt):
    K, N = 128, 48
    d = syn.custom_layer(21, 8, K, N)
    Xc = _orthogonal_calibration(K)
    rtn = o.prepare(d["W"], d["bias"], Xc, fmt=fmt)
    gq = o.prepare(d["W"], d["bias"], Xc, fmt=fmt, method="gptq")
    U = gq["gptq_U"]
    assert np.count_nonzero(np.triu(U, 1)) == 0
    np.testing.assert_array_equal(gq["w_codes"], rtn["w_codes"])
    np.testing.assert_array_equal(gq["w_scales"], rtn["w_scales"])
    np.testing.assert_array_equal(gq["w_deq"], rtn["w_deq"])


def _obs_brute_force(R, H, fmt, g_exp):
    """Greedy Optimal Brain Surgeon in the fixed order k = 0, 1, ...: with F the
    coordinates not yet fixed (k included), quantize w_k and move w_F by
    -(w_k - q_k) [H_F^-1]_{:,k} / [H_F^-1]_kk, H_F^-1 inverted afresh."""
    K, N = R.shape
    G = 16 if fmt == "nvfp4" else 64
    codes = np.zeros((N, K), dtype=np.int64)
    fed = np.zeros((N, K))
    inv_F = [np.linalg.inv(H[k:, k:]) for k in range(K)]
    for n in range(N):
        w = R[:, n].astype(np.float64).copy()
        for k in range(K):
            if k % G == 0:
                a = np.max(np.abs(w[k:k + G].astype(F32)))
                s, inv = o.nvfp4_group_scale(np.array([a]), g_exp) if fmt == "nvfp4" else o.int4_group_scale(np.array([a]))
            fed[n, k] = w[k]
            v = np.array([w[k]]).astype(F32)
            if fmt == "nvfp4":
                c = o.nvfp4_codes(v, s, inv)
                q = float(o.e2m1_decode(c)[0] * s[0] * 2.0 ** g_exp)
            else:
                c = o.int4_codes(v, inv)
                q = float(c[0]) * float(s[0])
            codes[n, k] = int(c[0])
            Hi = inv_F[k]
            w[k:] -= (w[k] - q) / Hi[0, 0] * Hi[:, 0]
    return codes, fed


@pytest.mark.parametrize("fmt,K", [("nvfp4", 48), ("int4", 128)])
def test_matches_brute_force_obs(fmt, K):
    d = syn.custom_layer(22, 8, K, 16, latent_rank=4, calib_tokens=96)
    lam, inv = o.smoothing_factors(d["Xc"], d["W"])
    R = o.fp32(lam.astype(np.float64)[:, None] * d["W"].astype(np.float64))
    H = o.gptq_hessian(d["Xc"], inv)
    g_exp = o.weight_tensor_exponent(R) if fmt == "nvfp4" else 0
    N = 5
    R = R[:, :N]
    q = o.gptq_quantize(R, o.gptq_factor(H), fmt, g_exp if fmt == "nvfp4" else None)
    codes, fed = _obs_brute_force(R, H, fmt, g_exp)
    got = q["w_codes"].astype(np.int64)
    np.testing.assert_array_equal(got, codes)
    np.testing.assert_allclose(q["w_fed"], fed, rtol=1e-9, atol=1e-12)
    # the error feedback moved the values: this is not round-to-nearest
    assert np.max(np.abs(fed - R.T)) > 1e-3 * np.max(np.abs(R))


@pytest.mark.parametrize("fmt", ["nvfp4", "int4"])
def test_lowers_output_error_on_correlated_activations(fmt):
    d = syn.custom_layer(7, 64, 256, 128, latent_rank=8, calib_tokens=512, with_heldout=True)
    rtn = o.prepare(d["W"], d["bias"], d["Xc"], fmt=fmt)
    gq = o.prepare(d["W"], d["bias"], d["Xc"], fmt=fmt, method="gptq")
    np.testing.assert_array_equal(gq["R"], rtn["R"])        # same residual, another quantizer

    def err(p, X):
        Xs = o.smoothed_activations(X, p["inv_lam"]).astype(np.float64)
        return np.linalg.norm(Xs @ (p["R"].astype(np.float64) - p["w_deq"].T))

    assert err(gq, d["Xc"]) < 0.6 * err(rtn, d["Xc"])
    assert err(gq, d["Xh"]) < 0.75 * err(rtn, d["Xh"])
