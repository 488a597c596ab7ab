"""GPU parity of the CUDA path against the CPU oracle, through the C ABI.

Bar (SVDQuant W4A4 layer): activation and weight codes and scales bit-exact on
shared inputs; BF16 outputs within relative Frobenius 2e-3 and max-abs
1e-2 * max|Y| of the oracle's BF16-rounded output, the oracle rounding XL to
BF16 as the GPU does.
"""
import numpy as np
import pytest

import synthetic as syn
from oracle import svdq_oracle as o

import w4a4_diffusion_transformer_b200 as lib
from gpu_util import (assert_close_bf16, oracle_prep_from, prepare_gpu, run_forward, run_quantize,
                      unit_smoothing_layer)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def gpu():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from w4a4_diffusion_transformer_b200 import build
    build.build()
    lib.load()


def check_k1(L, X, mode=0):
    p = oracle_prep_from(L)
    got = run_quantize(L, X, mode)
    M, K = X.shape
    if mode in (0, 1):
        ref = o.quantize_activations(X, p["inv_lam"], "nvfp4", p["g_x_exp"])
        np.testing.assert_array_equal(got["scales"], ref["scale_bytes"])
        np.testing.assert_array_equal(got["codes"], o.pack_nibbles(ref["codes"]))
        # padding rows of the last 128-row block carry zero scales
        pad = (M + 127) // 128 * 128
        if pad > M:
            full = L.act_scales_to_logical(got["scales_dev"], pad)
            assert np.all(full[M:] == 0)
    if mode in (0, 2) and p["rank"] > 0:
        ref_xl = o.down_projection(X, p["L1d"])
        # fp32 accumulation on the GPU vs float64 here: a BF16 rounding may flip by one unit
        np.testing.assert_allclose(got["xl"], ref_xl, rtol=2 ** -7, atol=1e-6 * np.max(np.abs(ref_xl)))
    return got


# ---------------------------------------------------------------- K1

def test_k1_tiny_bit_exact():
    d = syn.layer("tiny")
    L = prepare_gpu(d)
    check_k1(L, d["X"])


@pytest.mark.parametrize("M,K", [(1, 64), (33, 128), (200, 320), (333, 576), (130, 1024)])
def test_k1_ragged_shapes(M, K):
    d = syn.custom_layer(M + K, M=M, K=K, N=64)
    L = prepare_gpu(d)
    check_k1(L, d["X"])


@pytest.mark.parametrize("mode", [1, 2])
def test_k1_split_modes(mode):
    d = syn.custom_layer(11, M=160, K=512, N=64)
    L = prepare_gpu(d)
    check_k1(L, d["X"], mode)


def test_k1_edge_values():
    # smoothing factors are exactly 1, so the quantizer sees X itself
    K = 256
    d = unit_smoothing_layer(21, K, 64)
    L = prepare_gpu(d)
    assert np.all(L.export("lambda") == 1.0)
    g = 2.0 ** L.info["g_x_exp"]
    X = np.zeros((16, K), dtype=np.float32)
    # row 0: zeros.  row 1: far below the smallest scale -> zero scale, +0 codes
    X[1, :] = 1e-30
    # row 2: a = 6g -> s = 1, q = v / g: every E2M1 tie and signed zero
    X[2, :16] = np.array([6, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5, -0.25, -0.75, -5, -0.1, 0.1, 3, -6, 0]) * g
    # row 3: E4M3 scale ties: a = 6.375 g -> t = 1.0625 (tie 1.0 / 1.125); 7.125 g -> 1.1875
    X[3, 0] = 6.375 * g
    X[3, 16] = 7.125 * g
    X[3, 1:16] = np.linspace(-6, 6, 15) * g
    # row 4: subnormal scales (t < 2^-6)
    X[4, :16] = np.linspace(-1, 1, 16) * 6 * g * 2.0 ** -8 * 1.3
    X[4, 16:32] = np.linspace(-1, 1, 16) * 6 * g * 2.0 ** -11
    # row 5: saturating scale (t > 448) and saturating codes
    X[5, :16] = np.linspace(-1, 1, 16) * 6 * g * 600
    # rows 6-15: random with mixed magnitudes
    rng = np.random.default_rng(5)
    X[6:] = rng.standard_normal((10, K)) * g * 10.0 ** rng.uniform(-3, 2, (10, 1))
    X = syn.to_bf16(X)
    check_k1(L, X)


# ---------------------------------------------------------------- forward

def check_forward(L, d, flags=0, gelu=False):
    p = oracle_prep_from(L)
    y = run_forward(L, d["X"], flags)
    ref = o.forward(p, d["X"], gelu=gelu)
    return assert_close_bf16(y, ref["Y_bf16"], "forward"), y, ref, p


def test_forward_tiny():
    d = syn.layer("tiny")
    L = prepare_gpu(d)
    (err, mx), y, ref, _ = check_forward(L, d)
    # the layer output also stays close to the unquantized float64 product
    exact = d["X"].astype(np.float64) @ d["W"] + d["bias"]
    assert np.linalg.norm(y - exact) / np.linalg.norm(exact) < 0.05


@pytest.mark.parametrize("M,K,N", [(1, 64, 16), (200, 320, 272), (129, 512, 512), (300, 768, 400),
                                   (513, 1024, 256)])
def test_forward_ragged_shapes(M, K, N):
    d = syn.custom_layer(M * 7 + N, M=M, K=K, N=N)
    L = prepare_gpu(d)
    check_forward(L, d)


def test_forward_gelu():
    d = syn.custom_layer(31, M=256, K=512, N=512)
    L = prepare_gpu(d)
    check_forward(L, d, lib.FWD_GELU, gelu=True)


def test_forward_unfused_matches():
    d = syn.custom_layer(32, M=300, K=512, N=512)
    L = prepare_gpu(d)
    check_forward(L, d, lib.FWD_UNFUSED)
    check_forward(L, d, lib.FWD_UNFUSED | lib.FWD_GELU, gelu=True)


def test_forward_no_branch_is_bare_w4a4():
    d = syn.custom_layer(33, M=256, K=512, N=256)
    L = prepare_gpu(d)
    p = oracle_prep_from(L)
    y = run_forward(L, d["X"], lib.FWD_NO_BRANCH)
    xq = o.quantize_activations(d["X"], p["inv_lam"], "nvfp4", p["g_x_exp"])
    ref = o.bf16_round(xq["deq"] @ p["w_deq"].T + p["bias"])
    assert_close_bf16(y, ref, "bare")


def test_forward_rank_zero():
    d = syn.custom_layer(34, M=128, K=256, N=128)
    L = prepare_gpu(d, rank=0)
    check_forward(L, d)


def test_forward_zero_input_gives_bias():
    d = syn.custom_layer(35, M=64, K=256, N=128)
    L = prepare_gpu(d)
    d = dict(d, X=np.zeros((64, 256), dtype=np.float32))
    y = run_forward(L, d["X"])
    np.testing.assert_array_equal(y, np.broadcast_to(o.bf16_round(L.export("bias")), y.shape))


def test_forward_zero_input_gelu_of_bias():
    # X = 0 makes the accumulator zero, so the GELU epilogue sees y = b exactly:
    # Y = bf16(GELU(b)) for a bias sweep over [-12, 12], within one BF16 ulp of
    # the float64 tanh form rounded once (the GPU evaluates it in float32), or
    # within 2^-122 (about 1.9e-37) where float32 runs out of range: for b below
    # about -10 the denominator 1 + e^(-2u) exceeds 2^126, the fast division
    # returns zero, and the true value is below 1.2e-37 in magnitude
    d = syn.custom_layer(38, M=64, K=256, N=512)
    b = syn.to_bf16(np.linspace(-12.0, 12.0, 512))
    d = dict(d, bias=b, X=np.zeros((64, 256), dtype=np.float32))
    L = prepare_gpu(d)
    y = run_forward(L, d["X"], lib.FWD_GELU)
    ref = o.bf16_round(o.gelu_tanh(b.astype(np.float64)))
    ulp = np.ldexp(1.0, np.frexp(np.maximum(np.abs(ref), 2.0 ** -126))[1] - 8)
    tol = np.maximum(ulp, 2.0 ** -122)
    assert np.all(np.abs(y - ref[None, :]) <= tol[None, :])
    assert np.mean(y == ref[None, :]) > 0.97


def test_forward_deterministic():
    d = syn.custom_layer(36, M=384, K=512, N=512)
    L = prepare_gpu(d)
    y1 = run_forward(L, d["X"])
    y2 = run_forward(L, d["X"])
    np.testing.assert_array_equal(y1, y2)


def test_independent_prepare_parity_tiny():
    # the oracle's own prepare (LAPACK SVD) against the library's end to end
    d = syn.layer("tiny")
    L = prepare_gpu(d)
    y = run_forward(L, d["X"])
    ref = o.forward(o.prepare(d["W"], d["bias"], d["Xc"]), d["X"])["Y_bf16"]
    assert_close_bf16(y, ref, "independent prepare")


def test_mlp_chain_fc1_gelu_fc2():
    # fc1 (GELU epilogue) feeds fc2: fc2's codes are checked bit-exact on the
    # GPU-produced BF16 input, the chain's output by tolerance
    M = 256
    d1 = syn.custom_layer(40, M=M, K=512, N=1024, sigma0=20.0)
    L1 = prepare_gpu(d1)
    p1 = oracle_prep_from(L1)
    h_gpu = run_forward(L1, d1["X"], lib.FWD_GELU)
    h_ref = o.forward(p1, d1["X"], gelu=True)["Y_bf16"]
    assert_close_bf16(h_gpu, h_ref, "fc1")
    # fc2: weights from the recipe, calibration = GELU(fc1) on fc1's calibration batch (oracle)
    d2 = syn.custom_layer(41, M=M, K=1024, N=512, sigma0=20.0, outliers=False)
    d2["Xc"] = o.forward(p1, d1["Xc"], gelu=True)["Y_bf16"].astype(np.float32)
    L2 = prepare_gpu(d2)
    check_k1(L2, h_gpu)
    y = run_forward(L2, h_gpu)
    ref = o.forward(oracle_prep_from(L2), h_gpu)["Y_bf16"]
    assert_close_bf16(y, ref, "fc2 on GPU input")
    ref_chain = o.forward(oracle_prep_from(L2), h_ref.astype(np.float32))["Y_bf16"]
    err = np.linalg.norm(y - ref_chain) / np.linalg.norm(ref_chain)
    assert err < 2e-2, err


@pytest.mark.slow
def test_attn_out_full_size_sampled_rows():
    # FLUX.1 attention output projection at full size (M=4608, K=N=3072), in
    # the launch configuration the benchmark times; the oracle checks a sample
    # of rows (codes, scales and outputs)
    d = syn.layer("attn_out")
    L = prepare_gpu(d)
    p = oracle_prep_from(L)
    X = d["X"]
    q = run_quantize(L, X)
    y = run_forward(L, X)
    rows = np.unique(np.concatenate([np.arange(0, 4608, 97), [4607, 4480, 4479]]))
    ref = o.quantize_activations(X[rows], p["inv_lam"], "nvfp4", p["g_x_exp"])
    np.testing.assert_array_equal(q["scales"][rows], ref["scale_bytes"])
    np.testing.assert_array_equal(q["codes"][rows], o.pack_nibbles(ref["codes"]))
    yref = o.forward(p, X[rows])["Y_bf16"]
    assert_close_bf16(y[rows], yref, "attn_out sampled rows")
    assert np.all(np.isfinite(y))


# ---------------------------------------------------------------- CTA-pair GEMM (selectable kernel)

def _prepare_with_kernel(d, kernel):
    import os
    old = os.environ.get("SVDQ_K2_KERNEL")
    os.environ["SVDQ_K2_KERNEL"] = kernel          # read when the layer is created
    try:
        return prepare_gpu(d)
    finally:
        if old is None:
            del os.environ["SVDQ_K2_KERNEL"]
        else:
            os.environ["SVDQ_K2_KERNEL"] = old


@pytest.mark.parametrize("M,K,N,flags", [(200, 320, 272, 0), (513, 1024, 512, 0), (300, 768, 400, lib.FWD_GELU),
                                         (130, 512, 256, lib.FWD_NO_BRANCH)])
def test_pair_kernel_matches_oracle_and_single(M, K, N, flags):
    # 256 x 256 tiles on CTA pairs: same arithmetic as the single-CTA kernel,
    # so the two outputs agree bit for bit, and both meet the oracle's bar
    d = syn.custom_layer(M + 3 * N + K, M=M, K=K, N=N)
    Lp = _prepare_with_kernel(d, "pair")
    Ls = _prepare_with_kernel(d, "single")
    yp = run_forward(Lp, d["X"], flags)
    ys = run_forward(Ls, d["X"], flags)
    np.testing.assert_array_equal(yp.view(np.uint32), ys.view(np.uint32))
    p = oracle_prep_from(Lp)
    if flags & lib.FWD_NO_BRANCH:
        xq = o.quantize_activations(d["X"], p["inv_lam"], "nvfp4", p["g_x_exp"])
        ref = o.bf16_round(xq["deq"] @ p["w_deq"].T + p["bias"])
    else:
        ref = o.forward(p, d["X"], gelu=bool(flags & lib.FWD_GELU))["Y_bf16"]
    assert_close_bf16(yp, ref, "pair forward")
