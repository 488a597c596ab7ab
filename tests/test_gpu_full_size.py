"""GPU parity at the full FLUX.1 sizes the benchmark times, through the C ABI.

* the MLP pair at 4608 tokens: fc1 3072 -> 12288 with the GELU epilogue (48
  output tiles across N), then fc2 12288 -> 3072 on fc1's GPU output (48
  pipeline stages along K);
* the double-stream block at batch 4 (M = 18432 tokens, 144 row tiles): QKV
  3072 -> 9216, attention output 3072 -> 3072, fc1 3072 -> 12288 (GELU) and
  fc2 12288 -> 3072 on fc1's output, all NVFP4 with rank 32, plus the
  adaptive-norm W4A16 linear 3072 -> 18432 on 4 conditioning rows.

The whole output is produced on the GPU in the benchmark's launch
configuration; the oracle checks a sample of rows it can compute one by one:
seeded random rows plus the first and last rows and both sides of every
128-row tile boundary it picks.  Codes and scales must be bit-exact on those
rows, outputs within relative Frobenius 2e-3 and max-abs 1e-2 * max|Y| of the
oracle's BF16 output, and every output element must be finite.
"""
import numpy as np
import pytest

import synthetic as syn
from oracle import svdq_oracle as o

import w4a4_diffusion_transformer_b200 as lib
from gpu_util import assert_close_bf16, oracle_prep_from, prepare_gpu, to_numpy_f32

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module", autouse=True)
def gpu():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from w4a4_diffusion_transformer_b200 import build
    build.build()
    lib.load()


def sample_rows(M: int, seed: int, n: int = 40) -> np.ndarray:
    rng = np.random.default_rng([77, M, seed])
    picked = rng.choice(M, size=n, replace=False)
    edges = [0, 1, M - 1, M - 2]
    for r in picked[:6]:                       # both sides of a few tile boundaries
        b = (int(r) // 128) * 128
        edges += [b, max(b - 1, 0)]
    return np.unique(np.concatenate([picked, np.array(edges)]))


def run_device(L, x, flags=0):
    """K1 then K2 on device tensors, as the benchmark launches them; returns
    the device output and the host copies of codes and scales."""
    import torch
    M = x.shape[0]
    N = L.info["N"]
    stream = torch.cuda.current_stream()
    codes = torch.empty(L.act_code_bytes(M), dtype=torch.uint8, device="cuda")
    scales = torch.empty(L.act_scale_bytes(M), dtype=torch.uint8, device="cuda")
    xl = torch.empty((M, 32), dtype=torch.bfloat16, device="cuda")
    y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    L.quantize_act(x, M, codes, scales, xl, stream, 0)
    L.gemm(codes, scales, xl, M, y, stream, flags | lib.FWD_CHECK)
    torch.cuda.synchronize()
    return y, L.act_codes_to_logical(codes.cpu().numpy(), M), L.act_scales_to_logical(scales.cpu().numpy(), M)


def check_layer(L, x, rows, gelu=False, what=""):
    """Bit-exact codes and scales, and the output within tolerance, on `rows`."""
    import torch
    p = oracle_prep_from(L)
    y, codes, scales = run_device(L, x, lib.FWD_GELU if gelu else 0)
    assert bool(torch.isfinite(y).all()), f"{what}: non-finite output"
    Xr = to_numpy_f32(x[torch.from_numpy(rows).cuda()])
    ref = o.quantize_activations(Xr, p["inv_lam"], "nvfp4", p["g_x_exp"])
    np.testing.assert_array_equal(scales[rows], ref["scale_bytes"], err_msg=f"{what}: scales")
    np.testing.assert_array_equal(codes[rows], o.pack_nibbles(ref["codes"]), err_msg=f"{what}: codes")
    yr = to_numpy_f32(y[torch.from_numpy(rows).cuda()])
    assert_close_bf16(yr, o.forward(p, Xr, gelu=gelu)["Y_bf16"], what)
    return y, p


def fc2_layer(d1, p1, d2):
    """fc2 prepared on the oracle's GELU(fc1) of fc1's calibration batch."""
    d2 = dict(d2)
    d2["Xc"] = o.forward(p1, d1["Xc"], gelu=True)["Y_bf16"].astype(np.float32)
    return prepare_gpu(d2)


def test_mlp_pair_full_size_sampled_rows():
    from gpu_util import torch_bf16
    d1 = syn.layer("mlp", "fc1")
    M = d1["X"].shape[0]
    L1 = prepare_gpu(d1)
    x = torch_bf16(d1["X"])
    h, p1 = check_layer(L1, x, sample_rows(M, 1), gelu=True, what="fc1 4608x3072->12288 (GELU)")
    L2 = fc2_layer(d1, p1, syn.layer("mlp", "fc2"))
    check_layer(L2, h, sample_rows(M, 2), what="fc2 4608x12288->3072 on the GPU's fc1 output")


@pytest.mark.parametrize("name", ["qkv", "out"])
def test_block_b4_attention_linears_sampled_rows(name):
    from gpu_util import torch_bf16
    d = syn.layer("block_b4", name)
    M = d["X"].shape[0]
    assert M == 18432
    L = prepare_gpu(d)
    check_layer(L, torch_bf16(d["X"]), sample_rows(M, 3 + len(name)), what=f"block b4 {name}")


def test_block_b4_mlp_pair_sampled_rows():
    from gpu_util import torch_bf16
    d1 = syn.layer("block_b4", "fc1")
    M = d1["X"].shape[0]
    L1 = prepare_gpu(d1)
    h, p1 = check_layer(L1, torch_bf16(d1["X"]), sample_rows(M, 5), gelu=True, what="block b4 fc1 (GELU)")
    del d1["X"]
    L2 = fc2_layer(d1, p1, syn.layer("block_b4", "fc2"))
    check_layer(L2, h, sample_rows(M, 6), what="block b4 fc2 on the GPU's fc1 output")


def test_block_b4_adaln_w4a16():
    import torch
    from gpu_util import torch_bf16
    d = syn.layer("block_b4", "adaln", with_run=False)
    K, N = d["W"].shape
    X = syn.activations(4, 4, 4, K, syn.ROLE_X_RUN, outliers=False)
    L = prepare_gpu(d, fmt="w4a16", rank=0)
    y = torch.full((4, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    L.forward(torch_bf16(X), 4, y, None, 0, torch.cuda.current_stream(), lib.FWD_CHECK)
    torch.cuda.synchronize()
    ref = o.w4a16_forward(o.w4a16_prepare(d["W"], d["bias"]), X)["Y_bf16"]
    assert_close_bf16(to_numpy_f32(y), ref, "adaLN 4x3072->18432")


def test_mlp_chain_full_size_sampled_rows():
    """fc1 -> GELU -> fc2 through the chain at 4608 tokens: fc2's codes and
    scales from fc1's epilogue bit-exact on sampled rows against the oracle's
    quantizer on fc1's BF16 output (computed by a separate fc1 forward), XL2 and
    the output within tolerance, every output element finite."""
    import torch
    from gpu_util import torch_bf16
    d1 = syn.layer("mlp", "fc1")
    M = d1["X"].shape[0]
    L1 = prepare_gpu(d1)
    p1 = oracle_prep_from(L1)
    L2 = fc2_layer(d1, p1, syn.layer("mlp", "fc2"))
    p2 = oracle_prep_from(L2)
    x = torch_bf16(d1["X"])
    h, _, _ = run_device(L1, x, lib.FWD_GELU)
    stream = torch.cuda.current_stream()
    codes = torch.empty(L2.act_code_bytes(M), dtype=torch.uint8, device="cuda")
    scales = torch.empty(L2.act_scale_bytes(M), dtype=torch.uint8, device="cuda")
    xl = torch.empty((M, 32), dtype=torch.bfloat16, device="cuda")
    wsb = lib.mlp_workspace_bytes(L1, L2, M)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    lib.mlp_fc1(L1, L2, x, M, codes, scales, xl, ws, wsb, stream, lib.FWD_GELU | lib.FWD_CHECK)
    y = torch.full((M, L2.info["N"]), float("nan"), dtype=torch.bfloat16, device="cuda")
    lib.mlp_forward(L1, L2, x, M, y, ws, wsb, stream, lib.FWD_GELU | lib.FWD_CHECK)
    torch.cuda.synchronize()
    assert bool(torch.isfinite(y).all())
    rows = sample_rows(M, 8)
    idx = torch.from_numpy(rows).cuda()
    hr = to_numpy_f32(h[idx])
    ref = o.quantize_activations(hr, p2["inv_lam"], "nvfp4", p2["g_x_exp"])
    np.testing.assert_array_equal(L2.act_scales_to_logical(scales.cpu().numpy(), M)[rows], ref["scale_bytes"])
    np.testing.assert_array_equal(L2.act_codes_to_logical(codes.cpu().numpy(), M)[rows], o.pack_nibbles(ref["codes"]))
    ref_xl = o.down_projection(hr, p2["L1d"])
    np.testing.assert_allclose(to_numpy_f32(xl[idx]), ref_xl, rtol=2 ** -7, atol=1e-6 * np.max(np.abs(ref_xl)))
    assert_close_bf16(to_numpy_f32(y[idx]), o.forward(p2, hr)["Y_bf16"], "chain fc2 output 4608x12288->3072")
