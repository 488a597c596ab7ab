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
