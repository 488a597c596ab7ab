"""LoRA adapters concatenated into the 16-bit low-rank branch without
re-quantization (SOTA-314 practice page, "Known implementations": the paper's
engine loads off-the-shelf LoRA adapters without re-quantization).

Oracle pins: the adapted branch is exactly the base branch plus
bf16(X A) bf16(scale B) (linearity of the concatenated factors, float64); a
zero B leaves the layer unchanged; the residual's codes and scales never
change; the adapted layer approximates X (W + scale A B) + b as well as the base
layer approximates X W + b.  Library (host side, no GPU work): the stored
factors bit-exact against the oracle's rounding, argument errors, removal.
"""
import numpy as np
import pytest

import synthetic as syn
from oracle import svdq_oracle as o

import w4a4_diffusion_transformer_b200 as lib


def _adapter(K, N, r, seed, gain=0.05):
    rng = np.random.default_rng([9000 + seed, K, N, r])
    A = syn.to_bf16(rng.standard_normal((K, r)) / np.sqrt(K))
    B = syn.to_bf16(rng.standard_normal((r, N)) * gain)
    return A, B


@pytest.mark.parametrize("fmt", ["nvfp4", "int4"])
def test_oracle_branch_linearity(fmt):
    d = syn.custom_layer(120, M=64, K=256, N=192)
    p = o.prepare(d["W"], d["bias"], d["Xc"], fmt=fmt)
    A, B = _adapter(256, 192, 16, 1)
    s = 0.75
    q = o.attach_lora(p, A, B, s)
    assert q["rank"] == 48 and q["lora_r"] == 16
    np.testing.assert_array_equal(q["w_codes"], p["w_codes"])
    np.testing.assert_array_equal(q["w_scales"], p["w_scales"])
    y0 = o.forward(p, d["X"])["Y"]
    y1 = o.forward(q, d["X"])["Y"]
    xa = o.bf16_round(d["X"].astype(np.float64) @ A.astype(np.float64))
    bs = o.bf16_round(B.astype(np.float64) * s)
    np.testing.assert_allclose(y1 - y0, xa @ bs, rtol=1e-9, atol=1e-9 * np.max(np.abs(y0)))
    # B = 0: the layer is unchanged
    z = o.attach_lora(p, A, np.zeros_like(B), s)
    np.testing.assert_allclose(o.forward(z, d["X"])["Y"], y0, rtol=0, atol=1e-12 * np.max(np.abs(y0)))


def test_oracle_rank_zero_layer_takes_an_adapter():
    d = syn.custom_layer(121, M=32, K=128, N=64)
    p = o.prepare(d["W"], d["bias"], d["Xc"], rank=0)
    A, B = _adapter(128, 64, 8, 2)
    q = o.attach_lora(p, A, B, 1.0)
    assert q["rank"] == 8
    y = o.forward(q, d["X"])["Y"] - o.forward(p, d["X"])["Y"]
    np.testing.assert_allclose(y, o.bf16_round(d["X"].astype(np.float64) @ A) @ o.bf16_round(B.astype(np.float64)),
                               rtol=1e-9, atol=1e-12)


def test_oracle_adapted_layer_tracks_adapted_weight():
    d = syn.custom_layer(122, M=128, K=512, N=256)
    p = o.prepare(d["W"], d["bias"], d["Xc"])
    A, B = _adapter(512, 256, 32, 3, gain=0.5)
    s = 0.5
    X = d["X"].astype(np.float64)
    base = X @ d["W"] + d["bias"]
    adapted = X @ (d["W"] + s * A.astype(np.float64) @ B.astype(np.float64)) + d["bias"]
    e0 = np.linalg.norm(o.forward(p, d["X"])["Y"] - base) / np.linalg.norm(base)
    e1 = np.linalg.norm(o.forward(o.attach_lora(p, A, B, s), d["X"])["Y"] - adapted) / np.linalg.norm(adapted)
    assert e1 < 1.5 * e0 + 1e-3


@pytest.fixture(scope="module")
def built():
    from w4a4_diffusion_transformer_b200 import build
    build.build()
    lib.load()


@pytest.mark.parametrize("fmt", ["nvfp4", "int4"])
def test_library_stores_the_oracle_factors(built, fmt):
    d = syn.custom_layer(123, M=16, K=256, N=128)
    L = lib.Layer.prepare(syn.bf16_bits(d["W"]), syn.bf16_bits(d["bias"]), syn.bf16_bits(d["Xc"]), fmt=fmt,
                          device=-1)
    codes0 = L.export("w_codes").copy()
    A, B = _adapter(256, 128, 12, 4)
    L.set_lora(syn.bf16_bits(A), syn.bf16_bits(B), 0.3)
    np.testing.assert_array_equal(L.export("lora_A"), syn.bf16_bits(A))
    want = o.bf16_round(B.astype(np.float64) * float(np.float32(0.3)))
    np.testing.assert_array_equal(L.export("lora_B"), syn.bf16_bits(want.astype(np.float32)))
    np.testing.assert_array_equal(L.export("w_codes"), codes0)          # nothing re-quantized
    L.set_lora(None, None)
    for name in ("lora_A", "lora_B"):
        with pytest.raises(lib.SvdqError):
            L.export(name)


def test_library_argument_errors(built):
    d = syn.custom_layer(124, M=16, K=128, N=64)
    L = lib.Layer.prepare(syn.bf16_bits(d["W"]), None, syn.bf16_bits(d["Xc"]), device=-1)
    A, B = _adapter(128, 64, 33, 5)
    with pytest.raises(lib.SvdqError) as e:
        L.set_lora(syn.bf16_bits(A), syn.bf16_bits(B), 1.0)           # rank 33
    assert e.value.status == lib.EUNSUPPORTED
    A, B = _adapter(128, 64, 4, 6)
    with pytest.raises(lib.SvdqError) as e:
        L.set_lora(syn.bf16_bits(A), syn.bf16_bits(B), float("inf"))
    assert e.value.status == lib.EINVAL
    assert lib.load().svdq_set_lora(L._h, -1, None, None, 1.0) == lib.EINVAL
    assert lib.load().svdq_set_lora(L._h, 4, None, None, 1.0) == lib.EINVAL
    W = lib.Layer.prepare(syn.bf16_bits(d["W"]), None, None, fmt="w4a16", rank=0, device=-1)
    with pytest.raises(lib.SvdqError) as e:
        W.set_lora(syn.bf16_bits(A), syn.bf16_bits(B), 1.0)
    assert e.value.status == lib.EUNSUPPORTED
