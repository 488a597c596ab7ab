"""W8A8 (rank 16 at 8 bits; SOTA-314 practice page, "Do this") on the host:
the library's INT8 residual codes and per-channel scales bit-exact against
the oracle's quantizer on the library's residual, the rank rules, the options
the format does not take, and the activation layouts converted back.
"""
import numpy as np
import pytest

import synthetic as syn
from oracle import svdq_oracle as o

import w4a4_diffusion_transformer_b200 as lib


@pytest.fixture(scope="module", autouse=True)
def built():
    from w4a4_diffusion_transformer_b200 import build
    build.build()
    lib.load()


def _prep(d, rank=16, fmt="w8a8", flags=0):
    return lib.Layer.prepare(syn.bf16_bits(d["W"]), syn.bf16_bits(d["bias"]), syn.bf16_bits(d["Xc"]), fmt=fmt,
                             rank=rank, device=-1, flags=flags)


@pytest.mark.parametrize("K,N", [(256, 128), (576, 208), (1024, 48)])
def test_weight_codes_and_scales_bit_exact(K, N):
    d = syn.custom_layer(400 + K, M=16, K=K, N=N)
    L = _prep(d)
    assert L.info["rank"] == 16
    q = o.quantize_weights(L.export("R"), "w8a8")
    np.testing.assert_array_equal(L.export("w_codes").view(np.int8), q["w_codes"])
    np.testing.assert_array_equal(L.export("w_scales"), q["w_scales"].astype(np.float32))
    # the branch is the rank-16 split of the oracle's own factors up to sign
    p = o.prepare(d["W"], d["bias"], d["Xc"], fmt="w8a8", rank=16)
    np.testing.assert_allclose(np.abs(L.export("sigma")), p["S"][:16], rtol=1e-6)


def test_rank_rules_and_unsupported_options():
    d = syn.custom_layer(410, M=16, K=256, N=64)
    with pytest.raises(lib.SvdqError) as e:
        _prep(d, rank=32)                                   # 8 bits take rank 16
    assert e.value.status == lib.EUNSUPPORTED
    with pytest.raises(lib.SvdqError) as e:
        _prep(d, rank=16, fmt="nvfp4")                      # 4 bits take rank 32
    assert e.value.status == lib.EUNSUPPORTED
    with pytest.raises(lib.SvdqError) as e:
        _prep(d, flags=lib.PREP_GPTQ)
    assert e.value.status == lib.EUNSUPPORTED
    L = _prep(d, rank=0)
    assert L.info["rank"] == 0
    L = _prep(d)
    rng = np.random.default_rng(1)
    with pytest.raises(lib.SvdqError) as e:
        L.set_lora(syn.bf16_bits(syn.to_bf16(rng.standard_normal((256, 4)))),
                   syn.bf16_bits(syn.to_bf16(rng.standard_normal((4, 64)))), 1.0)
    assert e.value.status == lib.EUNSUPPORTED


def test_activation_layouts_convert_back():
    # codes: tiled in 128-column stages of 128-byte rows, 16-byte chunk c of row r
    # at ((r / 128) * nst + k / 128) * 16384 + (r % 128) * 128 + ((c ^ (r % 8)) * 16)
    d = syn.custom_layer(411, M=16, K=320, N=64)
    L = _prep(d)
    M, K = 200, 320
    nst = (K + 127) // 128
    mpad = (M + 127) // 128 * 128
    rng = np.random.default_rng(2)
    logical = rng.integers(-127, 128, size=(M, K)).astype(np.int8)
    dev = np.zeros(L.act_code_bytes(M), dtype=np.uint8)
    assert dev.size == mpad * nst * 128
    for r in range(M):
        for k in range(K):
            c = (k % 128) // 16
            off = ((r // 128) * nst + k // 128) * 16384 + (r % 128) * 128 + ((c ^ (r % 8)) * 16) + k % 16
            dev[off] = np.uint8(logical[r, k].view(np.uint8))
    np.testing.assert_array_equal(L.act_codes_to_logical(dev, M), logical)
    # scales: [s_x (mpad floats) | 1/s_x (mpad floats)], the first M are the per-token scales
    assert L.act_scale_bytes(M) == 8 * mpad
    s = rng.uniform(0.01, 2.0, size=2 * mpad).astype(np.float32)
    np.testing.assert_array_equal(L.act_scales_to_logical(s.view(np.uint8), M), s[:M])
