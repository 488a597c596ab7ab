"""Checkpoints of prepared layers (svdq_serialize / svdq_deserialize), on the
host: every stored tensor and the layer info survive the round trip for each
format, with and without a LoRA adapter; damaged bytes are refused, both by
the checksum and, for bytes re-signed after the change, by the checks of
each field against the shape and format."""
import numpy as np
import pytest
from hypothesis import HealthCheck, given, settings, strategies as st

import synthetic as syn

import w4a4_diffusion_transformer_b200 as lib

KEPT = ["lambda", "inv_lambda", "sigma", "L1d", "L2b", "w_codes", "w_scales", "bias"]


@pytest.fixture(scope="module", autouse=True)
def built():
    from w4a4_diffusion_transformer_b200 import build
    build.build()
    lib.load()


def _layer(fmt, rank, lora=False):
    d = syn.custom_layer(800 + rank, M=8, K=256, N=128)
    L = lib.Layer.prepare(syn.bf16_bits(d["W"]), syn.bf16_bits(d["bias"]),
                          None if fmt == "w4a16" else syn.bf16_bits(d["Xc"]), fmt=fmt, rank=rank, device=-1)
    if lora:
        rng = np.random.default_rng(3)
        L.set_lora(syn.bf16_bits(syn.to_bf16(rng.standard_normal((256, 8)))),
                   syn.bf16_bits(syn.to_bf16(rng.standard_normal((8, 128)))), 0.5)
    return L


@pytest.mark.parametrize("fmt,rank,lora", [("nvfp4", 32, False), ("nvfp4", 32, True), ("int4", 32, True),
                                           ("nvfp4", 0, False), ("w4a16", 0, False), ("w8a8", 16, False)])
def test_round_trip(fmt, rank, lora):
    L = _layer(fmt, rank, lora)
    blob = L.serialize()
    assert blob[:4] == b"SVDQ"
    R = lib.Layer.deserialize(blob, device=-1)
    assert R.info == L.info
    for name in KEPT + (["lora_A", "lora_B"] if lora else []):
        n = lib.load().svdq_tensor_bytes(L._h, lib.TENSORS[name][0])
        assert lib.load().svdq_tensor_bytes(R._h, lib.TENSORS[name][0]) == n, name
        if n:                                        # rank 0 has no branch tensors
            np.testing.assert_array_equal(R.export(name), L.export(name), err_msg=name)
    # preparation-only intermediates are not part of a checkpoint
    for name in ("R", "L1", "L2"):
        assert lib.load().svdq_tensor_bytes(R._h, lib.TENSORS[name][0]) == 0
    assert R.serialize() == blob


def _fnv1a64(data: bytes) -> int:
    """FNV-1a, 64-bit (Fowler, Noll and Vo), from its published definition."""
    h = 0xCBF29CE484222325
    for b in data:
        h = ((h ^ b) * 0x100000001B3) & 0xFFFFFFFFFFFFFFFF
    return h


def _resign(blob: bytearray) -> bytes:
    """The bytes with their trailing checksum recomputed."""
    body = bytes(blob[:-8])
    return body + _fnv1a64(body).to_bytes(8, "little")


def test_checksum_is_fnv1a_of_the_rest():
    blob = _layer("int4", 32, lora=True).serialize()
    assert int.from_bytes(blob[-8:], "little") == _fnv1a64(blob[:-8])
    assert int.from_bytes(blob[4:8], "little") == 2                     # format version


def test_every_single_byte_change_is_refused():
    blob = _layer("nvfp4", 32).serialize()
    rng = np.random.default_rng(11)
    positions = sorted(set(range(0, 96)) | set(rng.integers(0, len(blob), 300).tolist()) |
                       set(range(len(blob) - 8, len(blob))))
    for pos in positions:
        bad = bytearray(blob)
        bad[pos] ^= 1 << int(rng.integers(0, 8))
        with pytest.raises(lib.SvdqError) as e:
            lib.Layer.deserialize(bytes(bad), device=-1)
        assert e.value.status == lib.EINVAL, pos


def test_damaged_bytes_are_refused():
    blob = bytearray(_layer("nvfp4", 32).serialize())
    for bad in (bytes(blob[:-1]), bytes(blob[:40]), b"XXXX" + bytes(blob[4:]), bytes(blob) + b"\0"):
        with pytest.raises(lib.SvdqError) as e:
            lib.Layer.deserialize(bad, device=-1)
        assert e.value.status == lib.EINVAL
    # fields that disagree with the shape or format, re-signed so that only the
    # field checks can refuse them
    assert lib.Layer.deserialize(_resign(bytearray(blob)), device=-1).info["K"] == 256
    for off, delta in ((8, 64), (12, 16), (16, 1), (20, 7), (32, 40)):   # K, N, rank, format, lora_r
        wrong = bytearray(blob)
        wrong[off:off + 4] = ((int.from_bytes(blob[off:off + 4], "little") + delta) % 2 ** 32).to_bytes(4, "little")
        with pytest.raises(lib.SvdqError) as e:
            lib.Layer.deserialize(_resign(wrong), device=-1)
        assert e.value.status == lib.EINVAL, off
    # an array's byte count that no longer matches its bytes
    hdr = 64
    wrong = bytearray(blob)
    n0 = int.from_bytes(blob[hdr:hdr + 8], "little")                    # lam: K floats
    assert n0 == 256 * 4
    wrong[hdr:hdr + 8] = (n0 - 4).to_bytes(8, "little")
    with pytest.raises(lib.SvdqError) as e:
        lib.Layer.deserialize(_resign(wrong), device=-1)
    assert e.value.status == lib.EINVAL


def test_chain_and_adapter_rules_on_host_only_layers():
    # the MLP chain needs device layers: host-only layers get no workspace and a state error
    d1 = syn.custom_layer(830, M=8, K=256, N=512)
    d2 = syn.custom_layer(831, M=8, K=512, N=256)
    L1 = lib.Layer.prepare(syn.bf16_bits(d1["W"]), None, syn.bf16_bits(d1["Xc"]), device=-1)
    L2 = lib.Layer.prepare(syn.bf16_bits(d2["W"]), None, syn.bf16_bits(d2["Xc"]), device=-1)
    assert lib.mlp_workspace_bytes(L1, L2, 8) == 0
    st = lib.load().svdq_mlp_forward(L1._h, L2._h, 16, 8, 16, 16, 1 << 20, None, 0)
    assert st == lib.ESTATE
    # an adapter on a host-only layer is stored and survives a checkpoint
    rng = np.random.default_rng(9)
    L1.set_lora(syn.bf16_bits(syn.to_bf16(rng.standard_normal((256, 4)))),
                syn.bf16_bits(syn.to_bf16(rng.standard_normal((4, 512)))), 2.0)
    R = lib.Layer.deserialize(L1.serialize(), device=-1)
    np.testing.assert_array_equal(R.export("lora_B"), L1.export("lora_B"))


@settings(max_examples=25, deadline=None, derandomize=True, suppress_health_check=list(HealthCheck))
@given(fmt=st.sampled_from(["nvfp4", "int4", "w8a8", "w4a16"]), kb=st.integers(1, 4), nb=st.integers(1, 12),
       seed=st.integers(0, 10 ** 6), lora_r=st.integers(0, 32), with_rank=st.booleans())
def test_round_trip_over_random_layers(fmt, kb, nb, seed, lora_r, with_rank):
    K, N = 64 * kb, 16 * nb
    rank = 0 if fmt == "w4a16" or not with_rank else (16 if fmt == "w8a8" else 32)
    d = syn.custom_layer(seed, M=4, K=K, N=N)
    L = lib.Layer.prepare(syn.bf16_bits(d["W"]), syn.bf16_bits(d["bias"]),
                          None if fmt == "w4a16" else syn.bf16_bits(d["Xc"]), fmt=fmt, rank=rank, device=-1)
    adapter = lora_r > 0 and fmt in ("nvfp4", "int4")
    if adapter:
        rng = np.random.default_rng(seed)
        L.set_lora(syn.bf16_bits(syn.to_bf16(rng.standard_normal((K, lora_r)))),
                   syn.bf16_bits(syn.to_bf16(rng.standard_normal((lora_r, N)))), 0.25)
    blob = L.serialize()
    R = lib.Layer.deserialize(blob, device=-1)
    assert R.info == L.info
    assert R.serialize() == blob
    for name in KEPT + (["lora_A", "lora_B"] if adapter else []):
        if lib.load().svdq_tensor_bytes(L._h, lib.TENSORS[name][0]):
            np.testing.assert_array_equal(R.export(name), L.export(name), err_msg=name)
