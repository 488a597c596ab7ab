"""CPU tests of the host truncated SVD behind the low-rank split.

NOTE-257 note page ("Key results"): L1 = U Sigma[:, :r], L2 = V^T[:r, :], and
by Eckart-Young the truncated SVD is the best rank-r reduction.  The library
computes it by block subspace iteration; on a flat spectrum around sigma_r the
iteration moves to the Gram matrix of the smaller side and returns to the
weight for its last step.  These cases (Gaussian weights: a Marchenko-Pastur
bulk with no gap at r) take that route in the tall, wide and square
orientation, and are checked against LAPACK:

* sigma_0..31 and the discarded energy ||W_hat - L1 L2||_F^2 = sum_{i>=32}
  sigma_i^2 (Eckart-Young);
* L2's rows orthonormal and L1's columns orthogonal with norms sigma_i;
* the prepared bytes do not depend on the number of host threads.
"""
import os
import subprocess
import sys

import numpy as np
import pytest

import synthetic as syn

import w4a4_diffusion_transformer_b200 as lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    from w4a4_diffusion_transformer_b200 import build
    build.build()
    lib.load()


def _flat_layer(seed, K, N, M=64):
    rng = np.random.default_rng(seed)
    W = syn.to_bf16(rng.standard_normal((K, N)) * 0.05)
    Xc = syn.to_bf16(rng.standard_normal((M, K)))
    return W, np.zeros(N, dtype=np.float32), Xc


def _prep(W, bias, Xc):
    return lib.Layer.prepare(syn.bf16_bits(W), syn.bf16_bits(bias), syn.bf16_bits(Xc), device=-1)


@pytest.mark.parametrize("K,N", [(1024, 256), (256, 1024), (384, 384)])
def test_flat_spectrum_against_lapack(K, N):
    W, bias, Xc = _flat_layer(K + 7 * N, K, N)
    L = _prep(W, bias, Xc)
    W_hat = L.export("lambda").astype(np.float64)[:, None] * W.astype(np.float64)
    S = np.linalg.svd(W_hat, compute_uv=False)
    assert S[32] / S[31] > 0.95                      # no gap at r: the slow case
    assert L.info["svd_iterations"] > 12
    sigma = L.export("sigma")
    np.testing.assert_allclose(sigma, S[:32], rtol=1e-8)
    L1, L2 = L.export("L1"), L.export("L2")
    tail_ref = np.sum(S[32:] ** 2)
    tail = np.linalg.norm(W_hat - L1 @ L2) ** 2
    assert abs(tail - tail_ref) <= 1e-9 * tail_ref
    assert abs(L.info["svd_tail_energy"] - tail_ref) <= 1e-9 * tail_ref
    np.testing.assert_allclose(L2 @ L2.T, np.eye(32), atol=1e-10)
    np.testing.assert_allclose(L1.T @ L1, np.diag(S[:32] ** 2), atol=1e-9 * S[0] ** 2)


_CHILD = r"""
import sys, hashlib
sys.path.insert(0, sys.argv[1])
import numpy as np
import synthetic as syn
import w4a4_diffusion_transformer_b200 as lib
rng = np.random.default_rng(41)
W = syn.to_bf16(rng.standard_normal((512, 256)) * 0.05)
Xc = syn.to_bf16(rng.standard_normal((64, 512)))
L = lib.Layer.prepare(syn.bf16_bits(W), syn.bf16_bits(np.zeros(256, dtype=np.float32)), syn.bf16_bits(Xc),
                      device=-1)
h = hashlib.sha256()
for name in ("L1", "L2", "sigma", "L1d", "L2b", "R", "w_codes", "w_scales"):
    h.update(np.ascontiguousarray(L.export(name)).tobytes())
h.update(repr((L.info["svd_iterations"], L.info["svd_tail_energy"])).encode())
print(h.hexdigest())
"""


def test_prepared_bytes_independent_of_thread_count():
    out = []
    for threads in (1, 3, 8):
        env = dict(os.environ, OMP_NUM_THREADS=str(threads))
        r = subprocess.run([sys.executable, "-c", _CHILD, ROOT], env=env, capture_output=True, text=True,
                           timeout=600, cwd=ROOT)
        assert r.returncode == 0, r.stderr
        out.append(r.stdout.strip())
    assert out[0] and out[0] == out[1] == out[2], out
