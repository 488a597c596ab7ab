"""A layer rebuilt from its checkpoint (svdq_serialize / svdq_deserialize)
computes the same bytes as the layer it was saved from, for each W4A4-family
format and with a LoRA adapter attached."""
import numpy as np
import pytest

import synthetic as syn

import w4a4_diffusion_transformer_b200 as lib
from gpu_util import prepare_gpu, run_forward

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def gpu():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from w4a4_diffusion_transformer_b200 import build
    build.build()
    lib.load()


@pytest.mark.parametrize("fmt,rank,lora", [("nvfp4", 32, True), ("int4", 32, False), ("w8a8", 16, False)])
def test_checkpoint_forward_is_identical(fmt, rank, lora):
    d = syn.custom_layer(900 + rank, M=200, K=512, N=272)
    L = prepare_gpu(d, fmt=fmt, rank=rank)
    if lora:
        rng = np.random.default_rng(4)
        L.set_lora(syn.bf16_bits(syn.to_bf16(rng.standard_normal((512, 16)) / 20)),
                   syn.bf16_bits(syn.to_bf16(rng.standard_normal((16, 272)) / 5)), 0.5)
    y = run_forward(L, d["X"])
    R = lib.Layer.deserialize(L.serialize(), device=0)
    np.testing.assert_array_equal(run_forward(R, d["X"]), y)
    np.testing.assert_array_equal(run_forward(R, d["X"], lib.FWD_GELU), run_forward(L, d["X"], lib.FWD_GELU))
