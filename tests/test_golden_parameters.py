"""The method's printed parameters (tests/golden/method_parameters.txt, cited
there) against the oracle's constants and the library's formats: the ranks
the library accepts per bit width, the group sizes and the scale widths of
both the oracle's quantizers and the library's prepared tensors."""
import os

import numpy as np
import pytest

import synthetic as syn
from oracle import svdq_oracle as o

import w4a4_diffusion_transformer_b200 as lib

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "method_parameters.txt")


def _params():
    out = {}
    for line in open(GOLDEN):
        line = line.split("#", 1)[0].strip()
        if line:
            k, v = (s.strip() for s in line.split("="))
            out[k] = int(v)
    return out


P = _params()


@pytest.fixture(scope="module", autouse=True)
def built():
    from w4a4_diffusion_transformer_b200 import build
    build.build()
    lib.load()


def test_fixture_is_complete():
    assert set(P) == {"rank_at_4_bits", "rank_at_8_bits", "int4_group", "int4_scale_bits", "nvfp4_group",
                      "nvfp4_scale_bits"}


def test_oracle_groups_and_scale_widths():
    assert o.NVFP4_GROUP == P["nvfp4_group"] and o.INT4_GROUP == P["int4_group"]
    rng = np.random.default_rng(1)
    v = syn.to_bf16(rng.standard_normal((3, 256))).astype(np.float32)
    q = o.nvfp4_quantize(v, 0)
    assert q["codes"].shape == (3, 256) and q["scale_bytes"].shape == (3, 256 // P["nvfp4_group"])
    assert q["scale_bytes"].dtype.itemsize * 8 == P["nvfp4_scale_bits"]
    # each group of 16 has its own scale: changing one group moves only its scale
    v2 = v.copy()
    v2[0, :P["nvfp4_group"]] *= 4.0
    q2 = o.nvfp4_quantize(v2, 0)
    assert np.count_nonzero(q2["scale_bytes"] != q["scale_bytes"]) == 1
    qi = o.int4_quantize(v)
    assert qi["scales"].shape == (3, 256 // P["int4_group"])
    # 16-bit scales: every INT4 scale is a BF16 value
    s = np.asarray(qi["scales"], dtype=np.float64)
    np.testing.assert_array_equal(o.bf16_round(s), s)


@pytest.mark.parametrize("fmt,bits", [("nvfp4", 4), ("int4", 4), ("w8a8", 8)])
def test_library_ranks_per_bit_width(fmt, bits):
    d = syn.custom_layer(70, M=16, K=256, N=64)
    W, Xc = syn.bf16_bits(d["W"]), syn.bf16_bits(d["Xc"])
    rank = P["rank_at_4_bits"] if bits == 4 else P["rank_at_8_bits"]
    L = lib.Layer.prepare(W, None, Xc, fmt=fmt, rank=rank, device=-1)
    assert L.info["rank"] == rank
    other = P["rank_at_8_bits"] if bits == 4 else P["rank_at_4_bits"]
    with pytest.raises(lib.SvdqError) as e:
        lib.Layer.prepare(W, None, Xc, fmt=fmt, rank=other, device=-1)
    assert e.value.status == lib.EUNSUPPORTED
    assert lib.Layer.prepare(W, None, Xc, fmt=fmt, rank=0, device=-1).info["rank"] == 0


@pytest.mark.parametrize("fmt", ["nvfp4", "int4"])
def test_library_groups_and_scale_widths(fmt):
    K, N = 256, 64
    d = syn.custom_layer(71, M=16, K=K, N=N)
    L = lib.Layer.prepare(syn.bf16_bits(d["W"]), None, syn.bf16_bits(d["Xc"]), fmt=fmt, device=-1)
    g = P["nvfp4_group"] if fmt == "nvfp4" else P["int4_group"]
    bits = P["nvfp4_scale_bits"] if fmt == "nvfp4" else P["int4_scale_bits"]
    assert lib.load().svdq_tensor_bytes(L._h, lib.TENSORS["w_scales"][0]) * 8 == N * (K // g) * bits
    assert L.export("w_scales").shape == (N, K // g)
    assert L.act_scale_bytes(128) * 8 == 128 * (K // g) * bits        # activations: same groups, same widths
