"""Failure detection on the GPU without a fault: a kernel whose only wait can
never complete gives up after its budget, the layer's error word reports
SVDQ_ETIMEOUT through svdq_check, and the device stays usable."""
import numpy as np
import pytest

import synthetic as syn
from oracle import svdq_oracle as o

import w4a4_diffusion_transformer_b200 as lib
from gpu_util import assert_close_bf16, oracle_prep_from, prepare_gpu, run_forward

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def gpu():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from w4a4_diffusion_transformer_b200 import build
    build.build()
    lib.load()


def test_bounded_wait_expires_and_is_reported():
    import torch
    d = syn.layer("tiny")
    L = prepare_gpu(d)
    L.check()                                        # nothing pending
    s = torch.cuda.current_stream()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(s)
    L.selftest_wait_timeout(2000, s)                 # 2 ms budget, nothing ever arrives
    b.record(s)
    with pytest.raises(lib.SvdqError) as e:
        L.check(s)
    assert e.value.status == lib.ETIMEOUT
    assert a.elapsed_time(b) >= 1.9                  # the wait ran for its budget, then gave up
    L.check(s)                                       # the error word was cleared
    # the context is intact: the layer still meets the oracle's bar
    y = run_forward(L, d["X"])
    ref = o.forward(oracle_prep_from(L), d["X"])["Y_bf16"]
    assert_close_bf16(y, ref, "forward after a timeout")


def test_selftest_rejects_bad_budgets():
    d = syn.layer("tiny")
    L = prepare_gpu(d)
    for bad in (0, 10_000_001):
        with pytest.raises(lib.SvdqError) as e:
            L.selftest_wait_timeout(bad)
        assert e.value.status == lib.EINVAL
