"""GPU parity of the W8A8 variant (INT8 with one scale per token and per output
channel, rank-16 branch; SOTA-314 practice page, "Do this": rank 16 at 8 bits)
against the CPU oracle, through the C ABI.

Bar: activation codes and per-token scales bit-exact on shared inputs (the
library's exported 1/lambda); weight codes and scales bit-exact (host); BF16
outputs within relative Frobenius 2e-3 and max-abs 1e-2 * max|Y| of the
oracle's BF16-rounded output.  The integer products are exact (int32 on the
tensor cores), so only the FP32 epilogue and the BF16 rounding differ.
"""
import numpy as np
import pytest

import synthetic as syn
from oracle import svdq_oracle as o

import w4a4_diffusion_transformer_b200 as lib
from gpu_util import assert_close_bf16, oracle_prep_from, prepare_gpu, run_forward, run_quantize, to_numpy_f32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def gpu():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from w4a4_diffusion_transformer_b200 import build
    build.build()
    lib.load()


def _layer(M, K, N, seed, rank=16):
    d = syn.custom_layer(seed, M=M, K=K, N=N)
    return d, prepare_gpu(d, fmt="w8a8", rank=rank)


@pytest.mark.parametrize("M,K", [(1, 64), (33, 128), (200, 320), (333, 576), (130, 1024)])
def test_w8a8_k1_codes_and_scales_bit_exact(M, K):
    d, L = _layer(M, K, 64, 500 + M)
    p = oracle_prep_from(L)
    got = run_quantize(L, d["X"], 0)
    ref = o.quantize_activations(d["X"], p["inv_lam"], "w8a8")
    np.testing.assert_array_equal(got["scales"], ref["scales"].astype(np.float32))
    np.testing.assert_array_equal(got["codes"], ref["codes"])
    # padding rows: zero scales
    mpad = (M + 127) // 128 * 128
    sx = got["scales_dev"].view(np.float32)
    assert np.all(sx[M:mpad] == 0) and np.all(sx[mpad + M:] == 0)
    ref_xl = o.down_projection(d["X"], p["L1d"])
    np.testing.assert_allclose(got["xl"][:, :16], ref_xl, rtol=2 ** -7, atol=1e-6 * np.max(np.abs(ref_xl)))
    assert np.all(got["xl"][:, 16:] == 0)


@pytest.mark.parametrize("M,K,N", [(1, 64, 16), (200, 320, 272), (129, 512, 512), (300, 768, 400),
                                   (513, 1024, 256), (256, 3072, 3072)])
def test_w8a8_forward_parity(M, K, N):
    d, L = _layer(M, K, N, 600 + M + N)
    p = oracle_prep_from(L)
    y = run_forward(L, d["X"])
    assert_close_bf16(y, o.forward(p, d["X"])["Y_bf16"], f"w8a8 {M}x{K}->{N}")


def test_w8a8_gelu_unfused_rank_zero_zero_input_determinism():
    d, L = _layer(256, 512, 512, 701)
    p = oracle_prep_from(L)
    assert_close_bf16(run_forward(L, d["X"], lib.FWD_GELU), o.forward(p, d["X"], gelu=True)["Y_bf16"], "gelu")
    assert_close_bf16(run_forward(L, d["X"], lib.FWD_UNFUSED), o.forward(p, d["X"])["Y_bf16"], "unfused")
    y = run_forward(L, d["X"])
    np.testing.assert_array_equal(run_forward(L, d["X"]), y)
    X0 = np.zeros_like(d["X"])
    np.testing.assert_array_equal(run_forward(L, X0), np.broadcast_to(o.bf16_round(L.export("bias")), y.shape))
    d0, L0 = _layer(200, 256, 128, 702, rank=0)
    assert_close_bf16(run_forward(L0, d0["X"]), o.forward(oracle_prep_from(L0), d0["X"])["Y_bf16"], "rank 0")


@pytest.mark.slow
def test_w8a8_attn_out_full_size_sampled_rows():
    import torch
    from gpu_util import torch_bf16
    d = syn.layer("attn_out")
    M = d["X"].shape[0]
    L = prepare_gpu(d, fmt="w8a8", rank=16)
    p = oracle_prep_from(L)
    x = torch_bf16(d["X"])
    y = torch.full((M, 3072), float("nan"), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(L.workspace_bytes(M), dtype=torch.uint8, device="cuda")
    L.forward(x, M, y, ws, ws.numel(), torch.cuda.current_stream(), lib.FWD_CHECK)
    torch.cuda.synchronize()
    assert bool(torch.isfinite(y).all())
    rows = np.unique(np.concatenate([np.random.default_rng(9).choice(M, 40, replace=False), [0, 127, 128, M - 1]]))
    yr = to_numpy_f32(y[torch.from_numpy(rows).cuda()])
    assert_close_bf16(yr, o.forward(p, d["X"][rows])["Y_bf16"], "w8a8 attn-out 4608x3072->3072")
