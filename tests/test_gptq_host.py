"""The library's GPTQ residual quantizer (SVDQ_PREP_GPTQ) against the oracle,
on the host (svdq_prepare with device = -1 runs no GPU work).

SOTA-314 practice page, "Do this": the residual is quantized with GPTQ rather
than round-to-nearest.  Bar: codes and scales bit-exact against the oracle's
GPTQ run on shared inputs (the library's exported residual R and factor U);
the library's own U within 1e-10 of the oracle's, which factorises its own
Hessian of the same calibration batch.
"""
import numpy as np
import pytest
from hypothesis import HealthCheck, given, settings, strategies as st

import synthetic as syn
from oracle import svdq_oracle as o

import w4a4_diffusion_transformer_b200 as lib

GPTQ_KEEP = lib.PREP_GPTQ | lib.PREP_KEEP_GPTQ_FACTOR


@pytest.fixture(scope="module", autouse=True)
def built():
    from w4a4_diffusion_transformer_b200 import build
    build.build()
    lib.load()


def _prep(d, fmt, flags=GPTQ_KEEP, Xc=None, rank=32):
    Xc = d["Xc"] if Xc is None else Xc
    return lib.Layer.prepare(syn.bf16_bits(d["W"]), syn.bf16_bits(d["bias"]), syn.bf16_bits(Xc),
                             fmt=fmt, rank=rank, device=-1, flags=flags)


def _oracle_codes(L, fmt):
    q = o.gptq_quantize(L.export("R"), L.export("gptq_U"), fmt,
                        L.info["g_w_exp"] if fmt == "nvfp4" else None)
    if fmt == "nvfp4":
        return q, o.pack_nibbles(q["w_codes"]), q["w_scale_bytes"]
    return q, o.pack_nibbles(o.int4_nibbles(q["w_codes"])), syn.bf16_bits(q["w_scales"].astype(np.float32))


@pytest.mark.parametrize("fmt,K,N,latent", [("nvfp4", 256, 96, 8), ("int4", 256, 80, 8),
                                            ("nvfp4", 576, 208, 0), ("int4", 640, 48, 32)])
def test_codes_bit_exact_on_shared_factor(fmt, K, N, latent):
    d = syn.custom_layer(40 + K + N, 16, K, N, latent_rank=latent, calib_tokens=200)
    L = _prep(d, fmt)
    q, codes, scales = _oracle_codes(L, fmt)
    np.testing.assert_array_equal(L.export("w_codes"), codes)
    np.testing.assert_array_equal(L.export("w_scales"), scales)
    # the library's own factor matches the oracle's factorisation of its own Hessian
    Uo = o.gptq_factor(o.gptq_hessian(d["Xc"], L.export("inv_lambda")))
    U = L.export("gptq_U")
    assert np.max(np.abs(U - Uo)) <= 1e-10 * np.max(np.abs(Uo))
    # and GPTQ moved codes away from round-to-nearest
    rtn = o.quantize_weights(L.export("R"), fmt)
    assert np.mean(rtn["w_codes"] != q["w_codes"]) > 0.01


def test_dead_channel_and_rank_zero():
    # a calibration channel that is always zero takes the H_kk = 1 branch
    d = syn.custom_layer(47, 16, 128, 64, latent_rank=4, calib_tokens=64)
    Xc = d["Xc"].copy()
    Xc[:, 5] = 0.0
    Xc[:, 77] = 0.0
    for rank in (0, 32):
        L = _prep(d, "nvfp4", Xc=Xc, rank=rank)
        _, codes, scales = _oracle_codes(L, "nvfp4")
        np.testing.assert_array_equal(L.export("w_codes"), codes)
        np.testing.assert_array_equal(L.export("w_scales"), scales)
        Uo = o.gptq_factor(o.gptq_hessian(Xc, L.export("inv_lambda")))
        assert np.max(np.abs(L.export("gptq_U") - Uo)) <= 1e-10 * np.max(np.abs(Uo))


def test_lowers_output_error_through_the_library():
    d = syn.custom_layer(7, 64, 256, 128, latent_rank=8, calib_tokens=512, with_heldout=True)
    errs = {}
    for name, flags in (("rtn", 0), ("gptq", lib.PREP_GPTQ)):
        L = _prep(d, "nvfp4", flags=flags)
        p = {"inv_lam": L.export("inv_lambda"), "R": L.export("R")}
        codes = o.unpack_nibbles(L.export("w_codes"))
        sc = o.e4m3_decode(L.export("w_scales"))
        w_deq = o.e2m1_decode(codes) * np.repeat(sc, 16, axis=1) * 2.0 ** L.info["g_w_exp"]
        Xs = o.smoothed_activations(d["Xh"], p["inv_lam"]).astype(np.float64)
        errs[name] = np.linalg.norm(Xs @ (p["R"].astype(np.float64) - w_deq.T))
    assert errs["gptq"] < 0.75 * errs["rtn"]


def test_flags_validation():
    d = syn.custom_layer(48, 16, 128, 64, calib_tokens=64)
    with pytest.raises(lib.SvdqError) as e:
        _prep(d, "nvfp4", flags=0x4)                                     # unknown bit
    assert e.value.status == lib.EINVAL
    with pytest.raises(lib.SvdqError) as e:
        _prep(d, "nvfp4", flags=lib.PREP_KEEP_GPTQ_FACTOR)               # KEEP without GPTQ
    assert e.value.status == lib.EINVAL
    with pytest.raises(lib.SvdqError) as e:
        lib.Layer.prepare(syn.bf16_bits(d["W"]), None, None, fmt="w4a16", device=-1, flags=lib.PREP_GPTQ)
    assert e.value.status == lib.EINVAL
    # without KEEP the factor is not retained
    L = _prep(d, "nvfp4", flags=lib.PREP_GPTQ)
    assert lib.load().svdq_tensor_bytes(L._h, lib.TENSORS["gptq_U"][0]) == 0
    with pytest.raises(lib.SvdqError):
        L.export("gptq_U")
    # round-to-nearest layers have none either, and their codes did not change
    L0 = _prep(d, "nvfp4", flags=0)
    q = o.quantize_weights(L0.export("R"), "nvfp4")
    np.testing.assert_array_equal(L0.export("w_codes"), o.pack_nibbles(q["w_codes"]))



@settings(max_examples=20, deadline=None, derandomize=True, suppress_health_check=list(HealthCheck))
@given(fmt=st.sampled_from(["nvfp4", "int4"]), kb=st.integers(1, 6), nb=st.integers(1, 8),
       seed=st.integers(0, 10 ** 6), mcal=st.integers(8, 160), latent=st.sampled_from([0, 4, 16]),
       rank=st.sampled_from([0, 32]))
def test_codes_bit_exact_over_random_shapes(fmt, kb, nb, seed, mcal, latent, rank):
    # K and N span several factor blocks of 128 and ragged tails; calibration
    # batches both smaller and larger than K
    K, N = 64 * kb, 16 * nb
    d = syn.custom_layer(seed, 4, K, N, latent_rank=latent, calib_tokens=mcal)
    L = _prep(d, fmt, rank=rank)
    q, codes, scales = _oracle_codes(L, fmt)
    np.testing.assert_array_equal(L.export("w_codes"), codes)
    np.testing.assert_array_equal(L.export("w_scales"), scales)
    Uo = o.gptq_factor(o.gptq_hessian(d["Xc"], L.export("inv_lambda")))
    assert np.max(np.abs(L.export("gptq_U") - Uo)) <= 1e-10 * np.max(np.abs(Uo))
