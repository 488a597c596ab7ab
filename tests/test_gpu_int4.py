"""GPU parity of the INT4 variant (symmetric INT4 codes in groups of 64 with
BF16 scales; SOTA-314 practice page, "Do this") against the CPU oracle,
through the C ABI.

Bar: activation codes and scales bit-exact on shared inputs (the library's
exported 1/lambda); BF16 outputs within relative Frobenius 2e-3 and max-abs
1e-2 * max|Y| of the oracle's BF16-rounded output.
"""
import numpy as np
import pytest

import synthetic as syn
from oracle import svdq_oracle as o

import w4a4_diffusion_transformer_b200 as lib
from gpu_util import assert_close_bf16, oracle_prep_from, prepare_gpu, run_forward, run_quantize, unit_smoothing_layer

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def gpu():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from w4a4_diffusion_transformer_b200 import build
    build.build()
    lib.load()


def check_k1(L, X, mode=0, rows=None):
    p = oracle_prep_from(L)
    got = run_quantize(L, X, mode)
    M, K = X.shape
    if mode in (0, 1):
        sel = np.arange(M) if rows is None else rows
        ref = o.quantize_activations(X[sel], p["inv_lam"], "int4")
        np.testing.assert_array_equal(got["scales"][sel], syn.bf16_bits(ref["scales"]))
        np.testing.assert_array_equal(got["codes"][sel], o.pack_nibbles(o.int4_nibbles(ref["codes"])))
        # padding rows of the last 128-row block carry zero scales
        pad = (M + 127) // 128 * 128
        if pad > M:
            full = L.act_scales_to_logical(got["scales_dev"], pad)
            assert np.all(full[M:] == 0)
    if mode in (0, 2) and p["rank"] > 0 and rows is None:
        ref_xl = o.down_projection(X, p["L1d"])
        np.testing.assert_allclose(got["xl"], ref_xl, rtol=2 ** -7, atol=1e-6 * np.max(np.abs(ref_xl)))
    return got


def check_forward(L, X, flags=0, gelu=False):
    p = oracle_prep_from(L)
    y = run_forward(L, X, flags)
    ref = o.forward(p, X, gelu=gelu)
    return assert_close_bf16(y, ref["Y_bf16"], "int4 forward"), y, ref, p


# ---------------------------------------------------------------- K1 (INT4 quantizer)

def test_int4_k1_tiny_bit_exact():
    d = syn.layer("tiny")
    L = prepare_gpu(d, fmt="int4")
    check_k1(L, d["X"])


@pytest.mark.parametrize("M,K", [(1, 64), (33, 128), (200, 320), (333, 576), (130, 1024)])
def test_int4_k1_ragged_shapes(M, K):
    d = syn.custom_layer(M + 2 * K, M=M, K=K, N=64)
    L = prepare_gpu(d, fmt="int4")
    check_k1(L, d["X"])


@pytest.mark.parametrize("mode", [1, 2])
def test_int4_k1_split_modes(mode):
    d = syn.custom_layer(12, M=160, K=512, N=64)
    L = prepare_gpu(d, fmt="int4")
    check_k1(L, d["X"], mode)


def test_int4_k1_edge_values():
    # smoothing factors are exactly 1, so the quantizer sees X itself
    K = 256
    d = unit_smoothing_layer(22, K, 64)
    L = prepare_gpu(d, fmt="int4")
    assert np.all(L.export("lambda") == 1.0)
    X = np.zeros((16, K), dtype=np.float32)
    # row 1: a = 7 -> s = bf16(fp32(7 fp32(1/7))) = 1, q = v: every rounding tie, signed zeros
    X[1, :16] = [7, 0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 3.5, -3.5, 4.5, -6.5, 6.5, -0.0, 0.49, -7, 5.5]
    # row 2: a = 7 * 2^-20 (tiny scale); row 3: large values
    X[2, :64] = np.linspace(-1, 1, 64) * 7 * 2.0 ** -20
    X[3, :64] = np.linspace(-1, 1, 64) * 3.0e4
    # row 4: one group of zeros next to a nonzero group
    X[4, 64:128] = np.linspace(-2, 3, 64)
    # rows 5-15: random with mixed magnitudes
    rng = np.random.default_rng(6)
    X[5:] = rng.standard_normal((11, K)) * 10.0 ** rng.uniform(-3, 2, (11, 1))
    X = syn.to_bf16(X)
    got = check_k1(L, X)
    codes = o.unpack_nibbles(got["codes"])[1, :16]
    signed = np.where(codes >= 8, codes.astype(np.int64) - 16, codes)
    np.testing.assert_array_equal(signed, [7, 0, 2, 2, 0, -2, -2, 4, -4, 4, -6, 6, 0, 0, -7, 6])


# ---------------------------------------------------------------- forward (K1 + INT4 GEMM)

def test_int4_forward_tiny():
    d = syn.layer("tiny")
    L = prepare_gpu(d, fmt="int4")
    (err, mx), y, ref, _ = check_forward(L, d["X"])
    exact = d["X"].astype(np.float64) @ d["W"] + d["bias"]
    assert np.linalg.norm(y - exact) / np.linalg.norm(exact) < 0.1


@pytest.mark.parametrize("M,K,N", [(1, 64, 16), (200, 320, 272), (129, 512, 512), (300, 768, 400),
                                   (513, 1024, 256), (64, 3072, 528)])
def test_int4_forward_ragged_shapes(M, K, N):
    d = syn.custom_layer(M * 5 + N + 3, M=M, K=K, N=N)
    L = prepare_gpu(d, fmt="int4")
    check_forward(L, d["X"])


def test_int4_forward_gelu():
    d = syn.custom_layer(51, M=256, K=512, N=512)
    L = prepare_gpu(d, fmt="int4")
    check_forward(L, d["X"], lib.FWD_GELU, gelu=True)


def test_int4_forward_unfused_matches():
    d = syn.custom_layer(52, M=300, K=512, N=512)
    L = prepare_gpu(d, fmt="int4")
    check_forward(L, d["X"], lib.FWD_UNFUSED)


def test_int4_forward_no_branch_is_bare_w4a4():
    d = syn.custom_layer(53, M=256, K=512, N=256)
    L = prepare_gpu(d, fmt="int4")
    p = oracle_prep_from(L)
    y = run_forward(L, d["X"], lib.FWD_NO_BRANCH)
    xq = o.quantize_activations(d["X"], p["inv_lam"], "int4")
    ref = o.bf16_round(xq["deq"] @ p["w_deq"].T + p["bias"])
    assert_close_bf16(y, ref, "int4 bare")


def test_int4_forward_rank_zero():
    d = syn.custom_layer(54, M=128, K=256, N=128)
    L = prepare_gpu(d, fmt="int4", rank=0)
    check_forward(L, d["X"])


def test_int4_forward_zero_input_gives_bias():
    d = syn.custom_layer(55, M=64, K=256, N=128)
    L = prepare_gpu(d, fmt="int4")
    y = run_forward(L, np.zeros((64, 256), dtype=np.float32))
    np.testing.assert_array_equal(y, np.broadcast_to(o.bf16_round(L.export("bias")), y.shape))


def test_int4_forward_deterministic():
    d = syn.custom_layer(56, M=384, K=512, N=512)
    L = prepare_gpu(d, fmt="int4")
    np.testing.assert_array_equal(run_forward(L, d["X"]), run_forward(L, d["X"]))


def test_int4_weight_codes_bit_exact():
    d = syn.custom_layer(57, M=8, K=512, N=272)
    L = prepare_gpu(d, fmt="int4")
    q = o.quantize_weights(L.export("R"), "int4")
    np.testing.assert_array_equal(L.export("w_codes"), o.pack_nibbles(o.int4_nibbles(q["w_codes"])))
    np.testing.assert_array_equal(L.export("w_scales"), syn.bf16_bits(q["w_scales"]))


def test_int4_independent_prepare_parity_tiny():
    d = syn.layer("tiny")
    L = prepare_gpu(d, fmt="int4")
    y = run_forward(L, d["X"])
    ref = o.forward(o.prepare(d["W"], d["bias"], d["Xc"], fmt="int4"), d["X"])["Y_bf16"]
    assert_close_bf16(y, ref, "int4 independent prepare")


@pytest.mark.slow
def test_int4_qkv_full_size_sampled_rows():
    # INT4 fused QKV projection at full size (M=4608, K=3072 -> N=9216); the
    # oracle checks a sample of rows (codes, scales and outputs)
    d = syn.layer("qkv_int4")
    L = prepare_gpu(d, fmt="int4")
    p = oracle_prep_from(L)
    X = d["X"]
    rows = np.unique(np.concatenate([np.arange(0, 4608, 131), [4607, 4480, 4479]]))
    check_k1(L, X, rows=rows)
    y = run_forward(L, X)
    yref = o.forward(p, X[rows])["Y_bf16"]
    assert_close_bf16(y[rows], yref, "qkv int4 sampled rows")
    assert np.all(np.isfinite(y))


# ---------------------------------------------------------------- CTA-pair INT4 GEMM (selectable kernel)

def _prepare_int4_with_kernel(d, kernel):
    import os
    old = os.environ.get("SVDQ_K2_KERNEL")
    os.environ["SVDQ_K2_KERNEL"] = kernel          # read when the layer is created
    try:
        return prepare_gpu(d, fmt="int4")
    finally:
        if old is None:
            del os.environ["SVDQ_K2_KERNEL"]
        else:
            os.environ["SVDQ_K2_KERNEL"] = old


@pytest.mark.parametrize("M,K,N,flags", [(200, 320, 272, 0), (100, 512, 256, 0), (300, 768, 400, lib.FWD_GELU),
                                         (513, 1024, 512, 0)])
def test_int4_pair_kernel_matches_oracle_and_single(M, K, N, flags):
    # 256 x 256 tiles on CTA pairs (M = 100 and 200 leave the second CTA of the
    # last pair tile past the activation rows): same arithmetic as the
    # single-CTA kernel, so the outputs agree bit for bit, and both meet the bar
    d = syn.custom_layer(M + 5 * N + K, M=M, K=K, N=N)
    Lp = _prepare_int4_with_kernel(d, "pair")
    Ls = _prepare_int4_with_kernel(d, "single")
    yp = run_forward(Lp, d["X"], flags)
    ys = run_forward(Ls, d["X"], flags)
    np.testing.assert_array_equal(yp.view(np.uint32), ys.view(np.uint32))
    ref = o.forward(oracle_prep_from(Lp), d["X"], gelu=bool(flags & lib.FWD_GELU))["Y_bf16"]
    assert_close_bf16(yp, ref, "int4 pair forward")


# ---------------------------------------------------------------- range of the FP16 dequantization

def _int4_activation_exponent(Xc, inv_lam):
    # the layer's FP16 range exponent of the activation operand: the largest
    # smoothed calibration magnitude is moved to (2^7, 2^8]
    amax = float(np.max(np.abs(o.smoothed_activations(Xc, inv_lam))))
    return o.pow2_exponent_ceil(amax) - 8, amax


@pytest.mark.parametrize("gain", [64.0, 128.0, 1024.0])
def test_int4_activations_far_above_calibration(gain):
    # Rows of the run batch scaled by a power of two (exact in BF16) far above
    # anything in the calibration batch.  Up to about 220x the calibration
    # maximum every group is exact and the output meets the oracle's bar; a
    # group beyond that is clamped to the limit: the output stays finite and
    # equals the oracle's arithmetic with those group scales clamped.
    d = syn.custom_layer(60, M=256, K=512, N=384)
    L = prepare_gpu(d, fmt="int4")
    p = oracle_prep_from(L)
    X = d["X"].copy()
    hot = np.arange(0, 256, 17)
    X[hot] *= np.float32(gain)
    ex, calib_amax = _int4_activation_exponent(d["Xc"], p["inv_lam"])
    xq = o.quantize_activations(X, p["inv_lam"], "int4")
    limit = 8192.0 * 2.0 ** ex                          # the clamp, in scale units
    clamped = xq["scales"] > limit
    row_amax = float(np.max(np.abs(o.smoothed_activations(X[hot], p["inv_lam"]))))
    y = run_forward(L, X)
    assert np.all(np.isfinite(y))
    if gain <= 128.0:
        assert row_amax >= 0.25 * gain * calib_amax       # the rows really are far above calibration
        assert not clamped.any()
        assert_close_bf16(y, o.forward(p, X)["Y_bf16"], f"int4 x{gain:g}")
        return
    assert clamped.any() and row_amax > 220 * calib_amax
    K = X.shape[1]
    s_eff = np.minimum(xq["scales"], limit)
    deq = (xq["codes"].reshape(X.shape[0], K // 64, 64) * s_eff[:, :, None]).reshape(X.shape)
    model = o.forward(p, X, xq=dict(xq, deq=deq))["Y_bf16"]
    assert_close_bf16(y, model, f"int4 x{gain:g}, clamped groups")
    # rows without a clamped group still meet the oracle's own bar
    ok_rows = ~clamped.any(axis=1)
    assert ok_rows.sum() >= 200
    assert_close_bf16(y[ok_rows], o.forward(p, X[ok_rows])["Y_bf16"], "int4 rows without clamped groups")
