"""GPU parity of layers with a LoRA adapter in the low-rank branch
(svdq_set_lora; SOTA-314 practice page, "Known implementations": adapters
loaded without re-quantization).

Bar: BF16 outputs within relative Frobenius 2e-3 and max-abs 1e-2 * max|Y| of
the oracle's layer with the concatenated branch L1d' = [L1d | A],
L2b' = [L2b ; bf16(scale B)] (built from the library's exported tensors);
the residual's codes unchanged; XL_lora = bf16(X A) within the down
projection's tolerance; removing the adapter restores the base layer's output
bit for bit; the allocation-free forward gives the same bytes.
"""
import numpy as np
import pytest

import synthetic as syn
from oracle import svdq_oracle as o

import w4a4_diffusion_transformer_b200 as lib
from gpu_util import assert_close_bf16, oracle_prep_from, prepare_gpu, run_forward, run_quantize, torch_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def gpu():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from w4a4_diffusion_transformer_b200 import build
    build.build()
    lib.load()


def _adapter(K, N, r, seed, gain=0.2):
    rng = np.random.default_rng([9100 + seed, K, N, r])
    A = syn.to_bf16(rng.standard_normal((K, r)) / np.sqrt(K))
    B = syn.to_bf16(rng.standard_normal((r, N)) * gain)
    return A, B


def _with_lora(d, fmt, r, seed, scale=0.5, rank=32):
    L = prepare_gpu(d, fmt=fmt, rank=rank)
    K, N = d["W"].shape
    A, B = _adapter(K, N, r, seed)
    L.set_lora(syn.bf16_bits(A), syn.bf16_bits(B), scale)
    return L, A, B


@pytest.mark.parametrize("fmt,M,K,N,r", [("nvfp4", 200, 320, 272, 4), ("nvfp4", 513, 1024, 512, 32),
                                         ("nvfp4", 129, 768, 400, 16), ("int4", 200, 512, 272, 8),
                                         ("int4", 300, 1024, 384, 32)])
def test_lora_forward_parity(fmt, M, K, N, r):
    d = syn.custom_layer(200 + M + r, M=M, K=K, N=N)
    L, A, B = _with_lora(d, fmt, r, M)
    p = oracle_prep_from(L)
    assert p["rank"] == 32 + r
    y = run_forward(L, d["X"])
    assert_close_bf16(y, o.forward(p, d["X"])["Y_bf16"], f"{fmt} LoRA r={r}")
    # the adapter changed the output (it is not silently skipped)
    y0 = o.forward(oracle_prep_from(prepare_gpu(d, fmt=fmt)), d["X"])["Y_bf16"]
    assert np.linalg.norm(y - y0) > 10 * np.linalg.norm(y - o.forward(p, d["X"])["Y_bf16"])


@pytest.mark.parametrize("fmt", ["nvfp4", "int4"])
def test_lora_gelu_and_unfused(fmt):
    d = syn.custom_layer(231, M=256, K=512, N=512)
    L, A, B = _with_lora(d, fmt, 24, 31)
    p = oracle_prep_from(L)
    ref = o.forward(p, d["X"], gelu=True)["Y_bf16"]
    assert_close_bf16(run_forward(L, d["X"], lib.FWD_GELU), ref, f"{fmt} LoRA + GELU")
    assert_close_bf16(run_forward(L, d["X"], lib.FWD_GELU | lib.FWD_UNFUSED), ref, f"{fmt} LoRA unfused + GELU")
    assert_close_bf16(run_forward(L, d["X"], lib.FWD_UNFUSED), o.forward(p, d["X"])["Y_bf16"], f"{fmt} unfused")


def test_lora_on_rank_zero_layer_and_xl():
    d = syn.custom_layer(232, M=300, K=512, N=256)
    L, A, B = _with_lora(d, "nvfp4", 16, 32, rank=0)
    p = oracle_prep_from(L)
    assert_close_bf16(run_forward(L, d["X"]), o.forward(p, d["X"])["Y_bf16"], "rank 0 + LoRA")
    # XL columns 32..63 = bf16(X A), zero past r
    got = run_quantize(L, d["X"], 0)
    assert got["xl"].shape == (300, 64)
    ref = o.down_projection(d["X"], A.astype(np.float64))
    np.testing.assert_allclose(got["xl"][:, 32:48], ref, rtol=2 ** -7, atol=1e-6 * np.max(np.abs(ref)))
    assert np.all(got["xl"][:, 48:] == 0)


def test_lora_detach_restores_base_bit_for_bit_and_codes_unchanged():
    d = syn.custom_layer(233, M=384, K=768, N=512)
    L = prepare_gpu(d)
    codes = L.export("w_codes").copy()
    y_base = run_forward(L, d["X"])
    A, B = _adapter(768, 512, 20, 33)
    L.set_lora(syn.bf16_bits(A), syn.bf16_bits(B), 0.25)
    np.testing.assert_array_equal(L.export("w_codes"), codes)
    y_lora = run_forward(L, d["X"])
    assert not np.array_equal(y_lora, y_base)
    L.set_lora(None, None)
    np.testing.assert_array_equal(run_forward(L, d["X"]), y_base)


def test_lora_static_forward_and_chain_rejection():
    import torch
    d = syn.custom_layer(234, M=256, K=512, N=512)
    L, A, B = _with_lora(d, "nvfp4", 8, 34)
    y = run_forward(L, d["X"])
    ys = torch.full((256, 512), float("nan"), dtype=torch.bfloat16, device="cuda")
    L.forward_static(torch_bf16(d["X"]), 256, ys, torch.cuda.current_stream(), lib.FWD_CHECK)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(ys.float().cpu().numpy(), y)
    d2 = syn.custom_layer(235, M=256, K=512, N=256)
    L2 = prepare_gpu(d2)
    assert lib.mlp_workspace_bytes(L, L2, 256) == 0
    with pytest.raises(lib.SvdqError) as e:
        lib.mlp_forward(L, L2, torch_bf16(d["X"]), 256, torch.empty((256, 256), dtype=torch.bfloat16, device="cuda"),
                        torch.empty(1 << 22, dtype=torch.uint8, device="cuda"), 1 << 22)
    assert e.value.status == lib.EUNSUPPORTED
