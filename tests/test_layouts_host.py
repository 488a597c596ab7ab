"""The activation layouts the GEMMs read, as the ABI header documents them,
pinned on the host: a buffer built here from the documented formulas (written
independently of the library) must convert back to the logical arrays through
svdq_act_codes_to_logical / svdq_act_scales_to_logical, and the documented
sizes must match svdq_act_code_bytes / svdq_act_scale_bytes.  Host-only
layers (device -1), no GPU."""
import numpy as np
import pytest

import synthetic as syn
import w4a4_diffusion_transformer_b200 as lib


@pytest.fixture(scope="module", autouse=True)
def built():
    from w4a4_diffusion_transformer_b200 import build
    build.build()
    lib.load()


def _host_layer(M, K, N, fmt):
    d = syn.custom_layer(K + N, M=M, K=K, N=N)
    return lib.Layer.prepare(syn.bf16_bits(d["W"]), syn.bf16_bits(d["bias"]), syn.bf16_bits(d["Xc"]),
                             fmt=fmt, rank=32, device=-1)


SHAPES = [(1, 64, 32), (130, 320, 64), (200, 512, 48), (257, 1024, 16)]


@pytest.mark.parametrize("M,K,N", SHAPES)
def test_nvfp4_code_tiles(M, K, N):
    L = _host_layer(M, K, N, "nvfp4")
    rows_pad, nst = -(-M // 128) * 128, -(-K // 256)
    assert L.act_code_bytes(M) == rows_pad * nst * 128          # ceil(M/128)*128 * ceil(K/256) * 128
    rng = np.random.default_rng(M * 31 + K)
    logical = rng.integers(0, 256, size=(M, K // 2), dtype=np.uint8)
    dev = np.zeros(L.act_code_bytes(M), dtype=np.uint8)
    for r in range(M):
        for j in range(K // 2):
            t, jj = divmod(j, 128)                              # stage of 256 codes = 128 bytes of the row
            block = (r // 128) * nst + t
            dev[block * 16384 + (r % 128) * 128 + (((jj // 16) ^ (r % 8)) * 16) + jj % 16] = logical[r, j]
    np.testing.assert_array_equal(L.act_codes_to_logical(dev, M), logical)


@pytest.mark.parametrize("M,K,N", SHAPES)
def test_nvfp4_scale_chunks(M, K, N):
    # 512-byte chunk per (128-row block, 64-column block); inside it row r at
    # (r mod 32) * 16 + ((r / 32) mod 4) * 4, group g of the block at + g mod 4
    L = _host_layer(M, K, N, "nvfp4")
    rows_pad, kb = -(-M // 128) * 128, K // 64
    assert L.act_scale_bytes(M) == rows_pad // 128 * kb * 512
    rng = np.random.default_rng(M * 7 + K)
    logical = rng.integers(0, 256, size=(M, K // 16), dtype=np.uint8)
    dev = np.zeros(L.act_scale_bytes(M), dtype=np.uint8)
    for r in range(M):
        for g in range(K // 16):
            chunk = (r // 128) * kb + g // 4
            dev[chunk * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + g % 4] = logical[r, g]
    np.testing.assert_array_equal(L.act_scales_to_logical(dev, M), logical)


@pytest.mark.parametrize("M,K,N", SHAPES)
def test_int4_layouts(M, K, N):
    # codes row-major [M][K/2]; BF16 scales group-major [K/64][M rounded up to 128]
    L = _host_layer(M, K, N, "int4")
    rows_pad = -(-M // 128) * 128
    assert L.act_code_bytes(M) == M * K // 2
    assert L.act_scale_bytes(M) == rows_pad * (K // 64) * 2
    rng = np.random.default_rng(M + K * 3)
    codes = rng.integers(0, 256, size=(M, K // 2), dtype=np.uint8)
    np.testing.assert_array_equal(L.act_codes_to_logical(codes.ravel(), M), codes)
    scales = rng.integers(0, 65536, size=(M, K // 64), dtype=np.uint16)
    dev = np.zeros((K // 64, rows_pad), dtype=np.uint16)
    dev[:, :M] = scales.T
    np.testing.assert_array_equal(L.act_scales_to_logical(dev.view(np.uint8).ravel(), M), scales)
