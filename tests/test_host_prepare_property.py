"""Host preparation against the oracle over randomly drawn shapes and data
(hypothesis, derandomized: the same examples on every run).

For each format (NVFP4, INT4, W8A8), with K any multiple of 64 up to 512, N any
multiple of 16 up to 320 (so N may be below the rank), calibration batches of
1 to 64 tokens, with and without outlier channels and with weight spectra from
flat to strongly low-rank:

* lam and 1/lam bit-exact against the oracle's smoothing (SOTA-314 practice
  page, "Do this": smooth, then split);
* the stored branch factors are the BF16 roundings of the library's own
  float64 factors, L1d = bf16(diag(1/lam) L1) and L2b = bf16(L2);
* R = fp32(W_hat - diag(lam) L1d L2b) up to float64 summation order;
* the weight codes and scales bit-exact against the oracle's quantizer applied
  to the library's R, and the tensor-scale exponents equal to the oracle's.
"""
import numpy as np
import pytest
from hypothesis import HealthCheck, given, settings, strategies as st

import synthetic as syn
from oracle import svdq_oracle as o

import w4a4_diffusion_transformer_b200 as lib


@pytest.fixture(scope="module", autouse=True)
def built():
    from w4a4_diffusion_transformer_b200 import build
    build.build()
    lib.load()


@settings(max_examples=40, deadline=None, derandomize=True, suppress_health_check=list(HealthCheck))
@given(fmt=st.sampled_from(["nvfp4", "int4", "w8a8"]), kb=st.integers(1, 8), nb=st.integers(1, 20),
       seed=st.integers(0, 10 ** 6), mcal=st.integers(1, 64), outliers=st.booleans(),
       sigma0=st.sampled_from([0.0, 5.0, 40.0]))
def test_host_prepare_matches_the_oracle(fmt, kb, nb, seed, mcal, outliers, sigma0):
    K, N = 64 * kb, 16 * nb
    rank = 16 if fmt == "w8a8" else 32
    d = syn.custom_layer(seed, M=4, K=K, N=N, sigma0=sigma0, outliers=outliers, calib_tokens=mcal)
    L = lib.Layer.prepare(syn.bf16_bits(d["W"]), syn.bf16_bits(d["bias"]), syn.bf16_bits(d["Xc"]), fmt=fmt,
                          rank=rank, device=-1)
    lam, inv = o.smoothing_factors(d["Xc"], d["W"])
    np.testing.assert_array_equal(L.export("lambda"), lam)
    np.testing.assert_array_equal(L.export("inv_lambda"), inv)

    L1, L2 = L.export("L1"), L.export("L2")
    L1d = syn.from_bf16_bits(L.export("L1d")).astype(np.float64)
    L2b = syn.from_bf16_bits(L.export("L2b")).astype(np.float64)
    np.testing.assert_array_equal(L1d, o.bf16_round(inv.astype(np.float64)[:, None] * L1))
    np.testing.assert_array_equal(L2b, o.bf16_round(L2))

    W_hat = lam.astype(np.float64)[:, None] * d["W"].astype(np.float64)
    R_ref = o.fp32(W_hat - (lam.astype(np.float64)[:, None] * L1d) @ L2b)
    R = L.export("R")
    assert np.mean(R != R_ref) < 1e-3                      # a float64 sum in another order may flip a rounding
    np.testing.assert_allclose(R, R_ref, rtol=2 ** -23, atol=1e-30)

    q = o.quantize_weights(R, fmt)
    if fmt == "nvfp4":
        assert L.info["g_w_exp"] == q["g_w_exp"]
        assert L.info["g_x_exp"] == o.activation_tensor_exponent(d["Xc"], inv)
        np.testing.assert_array_equal(L.export("w_scales"), q["w_scale_bytes"])
        np.testing.assert_array_equal(L.export("w_codes"), o.pack_nibbles(q["w_codes"]))
    elif fmt == "int4":
        np.testing.assert_array_equal(L.export("w_codes"), o.pack_nibbles(o.int4_nibbles(q["w_codes"])))
        np.testing.assert_array_equal(syn.from_bf16_bits(L.export("w_scales")).astype(np.float64), q["w_scales"])
    else:
        np.testing.assert_array_equal(L.export("w_codes").view(np.int8), q["w_codes"])
        np.testing.assert_array_equal(L.export("w_scales"), q["w_scales"].astype(np.float32))
