"""CPU tests of the C ABI: the library loads and exports every declared
symbol, the host-side offline preparation agrees with the oracle, and the
argument checks reject bad input.  No GPU work is issued (layers are prepared
with device = -1)."""
import os
import re

import numpy as np
import pytest

import synthetic as syn
from oracle import svdq_oracle as o

import w4a4_diffusion_transformer_b200 as lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    from w4a4_diffusion_transformer_b200 import build
    build.build()
    lib.load()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "svdq.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(svdq_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported():
    L = lib.load()
    names = declared_functions()
    assert len(names) >= 13
    for n in names:
        assert hasattr(L, n), n
    assert sorted(lib.EXPORTED) == names


def _prep_host(d, fmt="nvfp4", rank=32):
    return lib.Layer.prepare(syn.bf16_bits(d["W"]), syn.bf16_bits(d["bias"]),
                             None if d.get("Xc") is None or fmt == "w4a16" else syn.bf16_bits(d["Xc"]),
                             fmt=fmt, rank=rank, device=-1)


@pytest.fixture(scope="module")
def tiny():
    d = syn.layer("tiny")
    return d, _prep_host(d), o.prepare(d["W"], d["bias"], d["Xc"])


def test_smoothing_bit_exact(tiny):
    d, L, p = tiny
    np.testing.assert_array_equal(L.export("lambda"), p["lam"])
    np.testing.assert_array_equal(L.export("inv_lambda"), p["inv_lam"])


def test_svd_eckart_young_and_subspace(tiny):
    d, L, p = tiny
    W_hat = p["lam"].astype(np.float64)[:, None] * d["W"]
    L1, L2 = L.export("L1"), L.export("L2")
    tail_lib = np.linalg.norm(W_hat - L1 @ L2) ** 2
    S = p["S"]
    tail_ref = np.sum(S[32:] ** 2)
    assert abs(tail_lib - tail_ref) <= 1e-4 * tail_ref
    assert abs(L.info["svd_tail_energy"] - tail_ref) <= 1e-4 * tail_ref
    np.testing.assert_allclose(L.export("sigma"), S[:32], rtol=1e-6)
    # the rank-32 product (sign-free) agrees with LAPACK's
    ref = p["L1"] @ p["L2"]
    assert np.linalg.norm(L1 @ L2 - ref) <= 1e-5 * np.linalg.norm(ref)


def test_branch_factors_and_residual_on_shared_inputs(tiny):
    d, L, p = tiny
    lam, inv = L.export("lambda"), L.export("inv_lambda")
    L1, L2 = L.export("L1"), L.export("L2")
    L1d = syn.from_bf16_bits(L.export("L1d")).astype(np.float64)
    L2b = syn.from_bf16_bits(L.export("L2b")).astype(np.float64)
    np.testing.assert_array_equal(L1d, o.bf16_round(inv.astype(np.float64)[:, None] * L1))
    np.testing.assert_array_equal(L2b, o.bf16_round(L2))
    W_hat = lam.astype(np.float64)[:, None] * d["W"]
    R_ref = o.fp32(W_hat - (lam.astype(np.float64)[:, None] * L1d) @ L2b)
    R = L.export("R")
    # float64 sums in a different order may flip a float32 rounding
    assert np.mean(R != R_ref) < 1e-3
    np.testing.assert_allclose(R, R_ref, rtol=2 ** -23, atol=1e-30)


def test_weight_codes_bit_exact_on_shared_residual(tiny):
    d, L, p = tiny
    q = o.quantize_weights(L.export("R"), "nvfp4")
    assert L.info["g_w_exp"] == q["g_w_exp"]
    np.testing.assert_array_equal(L.export("w_scales"), q["w_scale_bytes"])
    np.testing.assert_array_equal(L.export("w_codes"), o.pack_nibbles(q["w_codes"]))


def test_activation_tensor_scale(tiny):
    d, L, p = tiny
    assert L.info["g_x_exp"] == o.activation_tensor_exponent(d["Xc"], L.export("inv_lambda"))
    assert L.info["g_x_exp"] == p["g_x_exp"]


def test_independent_prepare_output_agrees(tiny):
    # library prepare vs oracle prepare, both evaluated by the oracle's forward
    d, L, p = tiny
    lp = dict(p)
    lp["L1d"] = syn.from_bf16_bits(L.export("L1d")).astype(np.float64)
    lp["L2b"] = syn.from_bf16_bits(L.export("L2b")).astype(np.float64)
    lp["inv_lam"] = L.export("inv_lambda")
    lp.update(o.quantize_weights(L.export("R"), "nvfp4"))
    lp["g_x_exp"] = L.info["g_x_exp"]
    y_lib = o.forward(lp, d["X"])["Y_bf16"]
    y_ref = o.forward(p, d["X"])["Y_bf16"]
    rel = np.linalg.norm(y_lib - y_ref) / np.linalg.norm(y_ref)
    assert rel <= 2e-3, rel
    assert np.max(np.abs(y_lib - y_ref)) <= 1e-2 * np.max(np.abs(y_ref))


def test_int4_prepare_bit_exact():
    d = syn.custom_layer(3, M=8, K=256, N=64, sigma0=10.0)
    L = _prep_host(d, fmt="int4")
    q = o.quantize_weights(L.export("R"), "int4")
    np.testing.assert_array_equal(L.export("w_codes"), o.pack_nibbles(o.int4_nibbles(q["w_codes"])))
    np.testing.assert_array_equal(syn.from_bf16_bits(L.export("w_scales")).astype(np.float64), q["w_scales"])


def test_w4a16_prepare_bit_exact():
    d = syn.custom_layer(4, M=4, K=128, N=64, outliers=False)
    L = _prep_host(d, fmt="w4a16")
    p = o.w4a16_prepare(d["W"], d["bias"])
    np.testing.assert_array_equal(L.export("w_codes"), o.pack_nibbles(o.int4_nibbles(p["w_codes"])))
    np.testing.assert_array_equal(syn.from_bf16_bits(L.export("w_scales")).astype(np.float64), p["w_scales"])
    np.testing.assert_array_equal(L.export("R"), d["W"].astype(np.float32))


def test_rank_zero_residual_is_smoothed_weight():
    d = syn.custom_layer(5, M=8, K=128, N=32)
    L = _prep_host(d, rank=0)
    lam = L.export("lambda").astype(np.float64)
    np.testing.assert_array_equal(L.export("R"), o.fp32(lam[:, None] * d["W"]))


def test_scale_layout_conversion():
    # the tensor-core scale layout: 512-byte chunks per (128-row block, 64-wide
    # K block); inside, row r at (r % 32) * 16 + ((r // 32) % 4) * 4, group g at + g % 4
    d = syn.custom_layer(6, M=8, K=256, N=32)
    L = _prep_host(d, rank=0)
    M, K = 200, 256
    nbytes = L.act_scale_bytes(M)
    assert nbytes == 2 * (K // 64) * 512
    dev = np.random.default_rng(0).integers(0, 255, nbytes, dtype=np.uint8)
    got = L.act_scales_to_logical(dev, M)
    for r in (0, 1, 31, 32, 77, 127, 128, 199):
        for g in range(K // 16):
            off = ((r // 128) * (K // 64) + g // 4) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + g % 4
            assert got[r, g] == dev[off]


def test_argument_errors():
    d = syn.custom_layer(7, M=8, K=128, N=32)
    W = syn.bf16_bits(d["W"])
    Xc = syn.bf16_bits(d["Xc"])
    with pytest.raises(lib.SvdqError) as e:
        lib.Layer.prepare(W[:, :24], None, Xc, device=-1)           # N % 16 != 0
    assert e.value.status == lib.EUNSUPPORTED
    with pytest.raises(lib.SvdqError) as e:
        lib.Layer.prepare(W[:96], None, Xc[:, :96], device=-1)      # K % 64 != 0
    assert e.value.status == lib.EUNSUPPORTED
    with pytest.raises(lib.SvdqError) as e:
        lib.Layer.prepare(W, None, None, device=-1)                 # W4A4 needs calibration
    assert e.value.status == lib.EINVAL
    with pytest.raises(lib.SvdqError) as e:
        lib.Layer.prepare(W, None, Xc, rank=17, device=-1)
    assert e.value.status == lib.EUNSUPPORTED
    L = lib.Layer.prepare(W, None, Xc, device=-1)
    with pytest.raises(lib.SvdqError) as e:                          # host-only layer: no forward
        L.forward(16, 8, 16, 256, 1 << 20)
    assert e.value.status == lib.ESTATE
    assert L.workspace_bytes(0) == 0


def test_activation_tensor_scale_exponent_range():
    # the first kernel's division-free reciprocal is pinned for activation
    # tensor-scale exponents in [-40, 30]; calibration batches outside are refused
    d = syn.custom_layer(8, M=8, K=128, N=32)
    W = syn.bf16_bits(d["W"])
    for scale in (2.0 ** 80, 2.0 ** -80):
        Xc = syn.bf16_bits(syn.to_bf16(d["Xc"].astype(np.float64) * scale))
        with pytest.raises(lib.SvdqError) as e:
            lib.Layer.prepare(W, None, Xc, device=-1)
        assert e.value.status == lib.EUNSUPPORTED
        L = lib.Layer.prepare(W, None, Xc, fmt="int4", device=-1)   # INT4 has no tensor scale
        L.close()
    for scale in (2.0 ** 20, 2.0 ** -20):                           # inside the range
        L = lib.Layer.prepare(W, None, syn.bf16_bits(syn.to_bf16(d["Xc"].astype(np.float64) * scale)), device=-1)
        assert -40 <= L.info["g_x_exp"] <= 30
        L.close()


def test_rank_above_matrix_rank():
    d = syn.custom_layer(8, M=4, K=64, N=16)
    L = _prep_host(d)
    L1, L2 = L.export("L1"), L.export("L2")
    assert np.all(np.isfinite(L1)) and np.all(np.isfinite(L2))
    assert np.all(L1[:, 16:] == 0) and np.all(L2[16:] == 0)
    lam = L.export("lambda").astype(np.float64)
    np.testing.assert_allclose(L1 @ L2, lam[:, None] * d["W"], rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("where", ["W", "bias", "calib"])
@pytest.mark.parametrize("bits", [0x7FC0, 0x7F80, 0xFF80])          # NaN, +inf, -inf
def test_prepare_refuses_non_finite_inputs(where, bits):
    import time
    d = syn.custom_layer(17, M=8, K=256, N=128)
    W, b, Xc = syn.bf16_bits(d["W"]).copy(), syn.bf16_bits(d["bias"]).copy(), syn.bf16_bits(d["Xc"]).copy()
    {"W": W, "bias": b, "calib": Xc}[where].reshape(-1)[37] = bits
    t = time.perf_counter()
    with pytest.raises(lib.SvdqError) as e:
        lib.Layer.prepare(W, b, Xc, device=-1)
    assert e.value.status == lib.EINVAL
    assert time.perf_counter() - t < 5.0                             # refused before any iteration
    if where == "calib":                                            # weight-only layers ignore the batch
        L = lib.Layer.prepare(W, b, Xc, fmt="w4a16", rank=0, device=-1)
        assert L.info["rank"] == 0


def test_device_argument():
    d = syn.custom_layer(19, M=8, K=128, N=64)
    args = (syn.bf16_bits(d["W"]), syn.bf16_bits(d["bias"]), syn.bf16_bits(d["Xc"]))
    blob = lib.Layer.prepare(*args, device=-1).serialize()
    for call in (lambda: lib.Layer.prepare(*args, device=-2), lambda: lib.Layer.deserialize(blob, device=-2)):
        with pytest.raises(lib.SvdqError) as e:
            call()
        assert e.value.status == lib.EINVAL


def test_device_placement_without_a_gpu_fails_cleanly():
    import torch
    if torch.cuda.is_available():
        pytest.skip("this machine has a GPU: placement succeeds")
    d = syn.custom_layer(20, M=8, K=128, N=64)
    args = (syn.bf16_bits(d["W"]), syn.bf16_bits(d["bias"]), syn.bf16_bits(d["Xc"]))
    blob = lib.Layer.prepare(*args, device=-1).serialize()
    for call in (lambda: lib.Layer.prepare(*args, device=0), lambda: lib.Layer.deserialize(blob, device=0)):
        with pytest.raises(lib.SvdqError) as e:
            call()
        assert e.value.status == lib.ECUDA


def test_operand_alignment_is_checked_before_the_layer_state():
    # raw addresses (never dereferenced: the host-only layer stops every call)
    d = syn.custom_layer(21, M=8, K=128, N=64)
    L = lib.Layer.prepare(syn.bf16_bits(d["W"]), None, syn.bf16_bits(d["Xc"]), device=-1)
    A, B = 0x10000, 0x10008                                     # 16-byte aligned / not
    for fn in (lambda x, y: L.forward(x, 8, y, 0x20000, 1 << 20), lambda x, y: L.forward_static(x, 8, y)):
        for x, y, want in ((A, A, lib.ESTATE), (B, A, lib.EINVAL), (A, B, lib.EINVAL)):
            with pytest.raises(lib.SvdqError) as e:
                fn(x, y)
            assert e.value.status == want, (hex(x), hex(y))
    for codes, scales, xl, want in ((A, A, A, lib.ESTATE), (B, A, A, lib.EINVAL), (A, B, A, lib.EINVAL),
                                    (A, A, B, lib.EINVAL)):
        with pytest.raises(lib.SvdqError) as e:
            L.quantize_act(A, 8, codes, scales, xl)
        assert e.value.status == want
        with pytest.raises(lib.SvdqError) as e:
            L.gemm(codes, scales, xl, 8, A)
        assert e.value.status == want
