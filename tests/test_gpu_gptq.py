"""GPU forward of layers whose residual was quantized by GPTQ
(SVDQ_PREP_GPTQ; SOTA-314 practice page, "Do this": the residual is quantized
with GPTQ rather than round-to-nearest), against the CPU oracle.

The forward kernels are the same as for round-to-nearest; what changes is the
prepared weight codes and scales.  Bar: the oracle's GPTQ on shared inputs
(the library's exported residual and factor) gives the weights; BF16 outputs
within relative Frobenius 2e-3 and max-abs 1e-2 * max|Y| of the oracle's
BF16-rounded output.  On correlated activations GPTQ's layer output is closer
to the unquantized product than round-to-nearest's.
"""
import numpy as np
import pytest

import synthetic as syn
from oracle import svdq_oracle as o

import w4a4_diffusion_transformer_b200 as lib
from gpu_util import assert_close_bf16, oracle_prep_from, run_forward

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def gpu():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from w4a4_diffusion_transformer_b200 import build
    build.build()
    lib.load()


def _prep(d, fmt, flags):
    return lib.Layer.prepare(syn.bf16_bits(d["W"]), syn.bf16_bits(d["bias"]), syn.bf16_bits(d["Xc"]),
                             fmt=fmt, device=0, flags=flags)


@pytest.mark.parametrize("fmt,M,K,N", [("nvfp4", 300, 768, 400), ("nvfp4", 513, 1024, 512),
                                       ("int4", 200, 512, 272), ("int4", 257, 1024, 384)])
def test_gptq_forward_parity(fmt, M, K, N):
    d = syn.custom_layer(60 + M, M, K, N, latent_rank=8, calib_tokens=384)
    L = _prep(d, fmt, lib.PREP_GPTQ | lib.PREP_KEEP_GPTQ_FACTOR)
    p = oracle_prep_from(L, gptq_U=L.export("gptq_U"))
    y = run_forward(L, d["X"])
    ref = o.forward(p, d["X"])
    assert_close_bf16(y, ref["Y_bf16"], f"{fmt} gptq forward")


@pytest.mark.parametrize("fmt", ["nvfp4", "int4"])
def test_gptq_output_closer_to_unquantized(fmt):
    d = syn.custom_layer(71, 512, 1024, 512, latent_rank=8, calib_tokens=512)
    exact = d["X"].astype(np.float64) @ d["W"].astype(np.float64) + d["bias"]
    errs = {}
    for name, flags in (("rtn", 0), ("gptq", lib.PREP_GPTQ)):
        y = run_forward(_prep(d, fmt, flags), d["X"])
        errs[name] = np.linalg.norm(y - exact) / np.linalg.norm(exact)
    assert errs["gptq"] < errs["rtn"], errs
