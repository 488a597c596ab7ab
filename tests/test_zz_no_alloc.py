"""The allocation-free forward (svdq_linear_forward_static): the same layer output
as svdq_linear_forward with a caller workspace, on two calls in a row, through
the C ABI.  Collected last on purpose (the file name), and self-contained so it
also passes alone in a fresh process."""
import numpy as np
import pytest

import synthetic as syn

import w4a4_diffusion_transformer_b200 as lib
from gpu_util import REL_FRO, MAX_ABS_FRAC, prepare_gpu, run_forward, to_numpy_f32, torch_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def gpu():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from w4a4_diffusion_transformer_b200 import build
    build.build()
    lib.load()


def test_static_workspace_forward_matches_caller_workspace_forward():
    import torch
    d = syn.custom_layer(90, M=1000, K=1024, N=768)
    L = prepare_gpu(d)
    M, N = 1000, 768
    assert L.workspace_bytes(M) <= lib.STATIC_WORKSPACE_BYTES
    y_ref = run_forward(L, d["X"])                     # existing entry point, caller workspace
    x = torch_bf16(d["X"])
    for call in range(2):                              # two calls in a row share the static array
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        L.forward_static(x, M, y, torch.cuda.current_stream(), lib.FWD_CHECK)
        torch.cuda.synchronize()
        got = to_numpy_f32(y).astype(np.float64)
        assert np.all(np.isfinite(got)), call
        err = np.linalg.norm(got - y_ref) / np.linalg.norm(y_ref)
        assert err <= REL_FRO, (call, err)
        assert np.max(np.abs(got - y_ref)) <= MAX_ABS_FRAC * np.max(np.abs(y_ref)), call
        # the same kernels on the same inputs: the same bytes, not only the same tolerance
        np.testing.assert_array_equal(got, y_ref)


def test_static_workspace_back_to_back_calls_on_one_stream():
    # Several calls queued on one stream with no synchronisation between them,
    # alternating two layers of different shapes: each call's first kernel
    # rewrites the shared array while the previous call's GEMM may still be
    # launching, so this checks that stream order protects the array.
    import torch
    da = syn.custom_layer(92, M=700, K=512, N=256)
    db = syn.custom_layer(93, M=1300, K=1024, N=512, sigma0=30.0)
    La, Lb = prepare_gpu(da), prepare_gpu(db)
    ref_a, ref_b = run_forward(La, da["X"]), run_forward(Lb, db["X"])
    xa, xb = torch_bf16(da["X"]), torch_bf16(db["X"])
    stream = torch.cuda.current_stream()
    outs = []
    for i in range(6):
        L, x, M, N = (La, xa, 700, 256) if i % 2 == 0 else (Lb, xb, 1300, 512)
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        L.forward_static(x, M, y, stream, 0)
        outs.append(y)
    torch.cuda.synchronize()
    La.check(stream)
    Lb.check(stream)
    for i, y in enumerate(outs):
        np.testing.assert_array_equal(to_numpy_f32(y), ref_a if i % 2 == 0 else ref_b)


def test_static_workspace_forward_of_a_weight_only_layer():
    # the adaptive-norm (W4A16) format needs no workspace and runs as the plain forward
    import torch
    d = syn.custom_layer(94, M=4, K=512, N=300, outliers=False)
    L = prepare_gpu(d, fmt="w4a16", rank=0)
    x = torch_bf16(d["X"])
    y_ref = torch.empty((4, 300), dtype=torch.bfloat16, device="cuda")
    L.forward(x, 4, y_ref, None, 0, torch.cuda.current_stream(), lib.FWD_CHECK)
    y = torch.full((4, 300), float("nan"), dtype=torch.bfloat16, device="cuda")
    L.forward_static(x, 4, y, torch.cuda.current_stream(), lib.FWD_CHECK)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(to_numpy_f32(y), to_numpy_f32(y_ref))


def test_static_workspace_rejects_sizes_beyond_its_limit():
    import torch
    d = syn.custom_layer(91, M=8, K=3072, N=256)
    L = prepare_gpu(d)
    M = 9350                                           # the first M that needs more than 16 MiB at K = 3072
    assert L.workspace_bytes(M) > lib.STATIC_WORKSPACE_BYTES
    x = torch.zeros((M, 3072), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((M, 256), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(lib.SvdqError) as e:
        L.forward_static(x, M, y, torch.cuda.current_stream(), 0)
    assert e.value.status == lib.EUNSUPPORTED
