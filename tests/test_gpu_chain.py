"""GPU parity of the fc1 -> fc2 chain (svdq_mlp_fc1 / svdq_mlp_forward): fc1's
GEMM epilogue hands fc2 its input already quantized.

The pages fuse the down projection with the quantizer because they read the
same input (SOTA-314 practice page, "Do this"; NOTE-257 note page, "Key
results"); in the MLP that input is fc1's GELU output.  Bar:

* fc2's activation codes and scales bit-exact against the oracle's quantizer
  applied to fc1's BF16 output as the GPU computes it (the same epilogue
  arithmetic, taken from a separate fc1 forward), and against the library's
  own first kernel on that output; padding rows zero;
* XL2 within the down projection's tolerance of the oracle's (the partial
  sums are added in a fixed order, so XL2 may differ from the first kernel's
  by a BF16 rounding);
* the chain's output within relative Frobenius 2e-3 and max-abs 1e-2 * max|Y|
  of the oracle's fc2 on that input; deterministic; the unfused measurement
  variant identical to two separate forwards.
"""
import numpy as np
import pytest

import synthetic as syn
from oracle import svdq_oracle as o

import w4a4_diffusion_transformer_b200 as lib
from gpu_util import assert_close_bf16, oracle_prep_from, prepare_gpu, run_forward, to_numpy_f32, torch_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def gpu():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from w4a4_diffusion_transformer_b200 import build
    build.build()
    lib.load()


def _pair(M, K, N1, N2, seed, rank1=32, rank2=32):
    d1 = syn.custom_layer(seed, M=M, K=K, N=N1, sigma0=20.0)
    L1 = prepare_gpu(d1, rank=rank1)
    p1 = oracle_prep_from(L1)
    d2 = syn.custom_layer(seed + 1, M=M, K=N1, N=N2, sigma0=20.0, outliers=False)
    d2["Xc"] = o.forward(p1, d1["Xc"], gelu=True)["Y_bf16"].astype(np.float32)
    L2 = prepare_gpu(d2, rank=rank2)
    return d1, L1, p1, L2


def _run_fc1(L1, L2, X, flags=lib.FWD_GELU):
    import torch
    M = X.shape[0]
    x = torch_bf16(X)
    codes = torch.full((L2.act_code_bytes(M),), 0xAB, dtype=torch.uint8, device="cuda")
    scales = torch.full((L2.act_scale_bytes(M),), 0xCD, dtype=torch.uint8, device="cuda")
    xl = torch.full((M, 32), float("nan"), dtype=torch.bfloat16, device="cuda")
    wsb = lib.mlp_workspace_bytes(L1, L2, M)
    assert wsb > 0
    ws = torch.full((wsb,), 0x7F, dtype=torch.uint8, device="cuda")
    lib.mlp_fc1(L1, L2, x, M, codes, scales, xl if L2.info["rank"] else None, ws, wsb,
                torch.cuda.current_stream(), flags | lib.FWD_CHECK)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), scales.cpu().numpy(), to_numpy_f32(xl)


def _run_mlp(L1, L2, X, flags=lib.FWD_GELU):
    import torch
    M = X.shape[0]
    x = torch_bf16(X)
    y = torch.full((M, L2.info["N"]), float("nan"), dtype=torch.bfloat16, device="cuda")
    wsb = lib.mlp_workspace_bytes(L1, L2, M, flags)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    lib.mlp_forward(L1, L2, x, M, y, ws, wsb, torch.cuda.current_stream(), flags | lib.FWD_CHECK)
    torch.cuda.synchronize()
    return to_numpy_f32(y)


def _check_fc2_input(L1, L2, X, gelu=True):
    """fc2's operands from the chain against the oracle and the first kernel on
    fc1's separately computed BF16 output."""
    import torch
    M = X.shape[0]
    h = run_forward(L1, X, lib.FWD_GELU if gelu else 0)            # fc1's BF16 output, same epilogue
    codes_d, scales_d, xl = _run_fc1(L1, L2, X, lib.FWD_GELU if gelu else 0)
    codes = L2.act_codes_to_logical(codes_d, M)
    scales = L2.act_scales_to_logical(scales_d, M)
    p2 = oracle_prep_from(L2)
    ref = o.quantize_activations(h, p2["inv_lam"], "nvfp4", p2["g_x_exp"])
    np.testing.assert_array_equal(scales[:M], ref["scale_bytes"])
    np.testing.assert_array_equal(codes[:M], o.pack_nibbles(ref["codes"]))
    pad = (M + 127) // 128 * 128
    if pad > M:
        full = L2.act_scales_to_logical(scales_d, pad)
        assert np.all(full[M:] == 0)
    # the library's first kernel on the same input writes the same bytes
    x = torch_bf16(h)
    c2 = torch.empty(L2.act_code_bytes(M), dtype=torch.uint8, device="cuda")
    s2 = torch.empty(L2.act_scale_bytes(M), dtype=torch.uint8, device="cuda")
    xl2 = torch.empty((M, 32), dtype=torch.bfloat16, device="cuda")
    L2.quantize_act(x, M, c2, s2, xl2, torch.cuda.current_stream(), 0 if L2.info["rank"] else 1)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(L2.act_codes_to_logical(c2.cpu().numpy(), M), codes)
    np.testing.assert_array_equal(L2.act_scales_to_logical(s2.cpu().numpy(), M), scales)
    if L2.info["rank"]:
        ref_xl = o.down_projection(h, p2["L1d"])
        np.testing.assert_allclose(xl, ref_xl, rtol=2 ** -7, atol=1e-6 * np.max(np.abs(ref_xl)))
    return h, p2


@pytest.mark.parametrize("M,K,N1,N2", [(300, 512, 768, 512), (129, 256, 320, 256), (1, 128, 1024, 64),
                                       (513, 768, 1536, 384)])
def test_chain_fc2_input_bit_exact(M, K, N1, N2):
    d1, L1, p1, L2 = _pair(M, K, N1, N2, seed=M + N1)
    _check_fc2_input(L1, L2, d1["X"])


def test_chain_without_gelu_and_rank_zero():
    d1, L1, p1, L2 = _pair(200, 256, 512, 256, seed=901, rank2=0)
    _check_fc2_input(L1, L2, d1["X"])
    d1, L1, p1, L2 = _pair(200, 256, 512, 256, seed=903, rank1=0)
    _check_fc2_input(L1, L2, d1["X"], gelu=False)


@pytest.mark.parametrize("M,K,N1,N2", [(300, 512, 768, 512), (640, 1024, 2048, 1024)])
def test_chain_forward_matches_oracle(M, K, N1, N2):
    d1, L1, p1, L2 = _pair(M, K, N1, N2, seed=7 * M)
    h, p2 = _check_fc2_input(L1, L2, d1["X"])
    y = _run_mlp(L1, L2, d1["X"])
    assert_close_bf16(y, o.forward(p2, h)["Y_bf16"], "chain on the GPU's fc1 output")
    # the unfused measurement variant is the two separate forwards, bit for bit
    yu = _run_mlp(L1, L2, d1["X"], lib.FWD_GELU | lib.FWD_UNFUSED)
    np.testing.assert_array_equal(yu, run_forward(L2, h))
    assert_close_bf16(y, yu, "chain vs separate layers")
    # deterministic
    np.testing.assert_array_equal(_run_mlp(L1, L2, d1["X"]), y)


def test_chain_rejects_mismatched_layers():
    import torch
    d1, L1, p1, L2 = _pair(64, 256, 512, 256, seed=911)
    d3 = syn.custom_layer(913, M=64, K=256, N=256)
    L3 = prepare_gpu(d3)                                  # K = 256 != fc1's N = 512
    L4 = prepare_gpu(syn.custom_layer(915, M=64, K=512, N=256), fmt="int4")
    for bad in (L3, L4):
        assert lib.mlp_workspace_bytes(L1, bad, 64) == 0
        with pytest.raises(lib.SvdqError) as e:
            lib.mlp_forward(L1, bad, torch_bf16(d1["X"]), 64, torch.empty((64, 256), dtype=torch.bfloat16,
                                                                             device="cuda"),
                            torch.empty(1 << 20, dtype=torch.uint8, device="cuda"), 1 << 20)
        assert e.value.status == lib.EUNSUPPORTED
    wsb = lib.mlp_workspace_bytes(L1, L2, 64)
    with pytest.raises(lib.SvdqError) as e:
        lib.mlp_forward(L1, L2, torch_bf16(d1["X"]), 64, torch.empty((64, 256), dtype=torch.bfloat16, device="cuda"),
                        torch.empty(wsb, dtype=torch.uint8, device="cuda"), wsb - 256)
    assert e.value.status == lib.EINVAL
