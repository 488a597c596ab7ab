"""GPU parity of the weight-only INT4 GEMV (the adaptive-normalization linears,
which stay W4A16 per the SOTA-314 practice page, "Do this") against the oracle."""
import numpy as np
import pytest

import synthetic as syn
from oracle import svdq_oracle as o

import w4a4_diffusion_transformer_b200 as lib
from gpu_util import assert_close_bf16, to_numpy_f32, torch_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def gpu():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from w4a4_diffusion_transformer_b200 import build
    build.build()
    lib.load()


def run_w4a16(W, b, X):
    import torch
    L = lib.Layer.prepare(syn.bf16_bits(W), syn.bf16_bits(b), None, fmt="w4a16", rank=0, device=0)
    M, K = X.shape
    N = W.shape[1]
    x = torch_bf16(X)
    y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    L.forward(x, M, y, None, 0, torch.cuda.current_stream(), lib.FWD_CHECK)
    torch.cuda.synchronize()
    return to_numpy_f32(y), L


@pytest.mark.parametrize("M,K,N", [(1, 64, 16), (4, 320, 272), (7, 1024, 520), (12, 512, 48), (16, 3072, 256),
                                   (20, 256, 40), (5, 12288, 64), (3, 64, 1)])
def test_w4a16_shapes(M, K, N):
    rng = np.random.default_rng(M * 1000 + K + N)
    W = syn.to_bf16(rng.standard_normal((K, N)) / np.sqrt(K))
    b = syn.to_bf16(rng.standard_normal(N) * 0.1)
    X = syn.to_bf16(rng.standard_normal((M, K)))
    y, L = run_w4a16(W, b, X)
    ref = o.w4a16_forward(o.w4a16_prepare(W, b), X)["Y_bf16"]
    assert_close_bf16(y, ref, f"w4a16 {M}x{K}x{N}")


def test_w4a16_adaln_full_size():
    # FLUX.1-dev adaptive-norm modulation linear: 4 conditioning rows, 3072 -> 18432
    d = syn.layer("block_b4", "adaln")
    X = syn.activations(4, 4, 4, 3072, syn.ROLE_X_RUN, outliers=False)
    y, L = run_w4a16(d["W"], d["bias"], X)
    ref = o.w4a16_forward(o.w4a16_prepare(d["W"], d["bias"]), X)["Y_bf16"]
    assert_close_bf16(y, ref, "adaLN")
    # codes and scales of the weights: bit-exact with the oracle
    p = o.w4a16_prepare(d["W"], d["bias"])
    np.testing.assert_array_equal(L.export("w_codes"), o.pack_nibbles(o.int4_nibbles(p["w_codes"])))
