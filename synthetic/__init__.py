"""Seeded synthetic inputs for the SVDQuant W4A4 linear layer.

This module is shared by the CPU oracle, the tests and the benchmark. It only
draws random numbers and rounds them to the layer's input dtype (BF16); it holds
none of the layer's own arithmetic (no smoothing, no SVD, no quantization, no
activation functions).

Stand-ins for FLUX.1 layers (SVDQuant, "What it buys" and "Key results" on the
practice and note pages): the pages measure on FLUX.1 models whose weights and
prompts are not available here, so every layer is a seeded synthetic matrix
with the shapes of a FLUX.1 double-stream block and the structure the method
relies on:

* activations X ~ N(0, 1) with 1% of the input channels (a fixed, seeded set)
  scaled by 50 -- the outlier channels that smoothing moves into the weights;
* weights W = N(0, 1/K) noise plus 32 rank-1 spikes sigma_i * u_i v_i^T with
  sigma_i = sigma0 * 0.85**i and orthonormal u_i, v_i -- a steep leading
  spectrum over a flat bulk (the "Figure 5" premise on the note page);
* bias ~ N(0, 0.02) (0.02 read as the variance, like the 1/K of the weights).

Every array is produced by ``numpy.random.default_rng([workload_id,
layer_id, role])`` in float64 and then rounded once to BF16 (round to nearest
even, through ``torch``'s cast).  Arrays are returned as float32 numpy arrays
whose values are exactly BF16-representable; ``bf16_bits`` gives the raw
16-bit patterns for the C ABI.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import numpy as np

# Roles of the random streams (the last entry of the seed sequence).
ROLE_W_NOISE = 0
ROLE_U = 1
ROLE_V = 2
ROLE_OUTLIERS = 3
ROLE_X_RUN = 4
ROLE_X_CALIB = 5
ROLE_BIAS = 6
ROLE_X_HELDOUT = 7
ROLE_X_LATENT = 8

CALIB_TOKENS = 256
SPIKES = 32
OUTLIER_FRACTION = 0.01
OUTLIER_GAIN = 50.0
SPIKE_DECAY = 0.85
BIAS_VARIANCE = 0.02
LATENT_NOISE = 0.5


@dataclasses.dataclass(frozen=True)
class LayerShape:
    """One linear layer: Y[M,N] = X[M,K] @ W[K,N] + b."""
    name: str
    M: int
    K: int
    N: int
    sigma0: float          # leading spike singular value
    fmt: str = "nvfp4"     # "nvfp4", "int4" (W4A4) or "w4a16"
    outliers: bool = True  # inject outlier channels into X
    layer_id: int = 0


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    workload_id: int
    layers: tuple
    description: str


def _wl(name, wid, desc, *layers):
    return Workload(name, wid, tuple(layers), desc)


# FLUX.1 hidden size 3072, MLP ratio 4, 4096 image + 512 text tokens.
WORKLOADS: Dict[str, Workload] = {
    w.name: w for w in [
        _wl("tiny", 0, "tiny SVDQuant linear 256x512->512, NVFP4 g16",
            LayerShape("tiny", 256, 512, 512, 20.0)),
        _wl("attn_out", 1, "FLUX.1 attention output projection 4608x3072->3072, NVFP4 g16",
            LayerShape("attn_out", 4608, 3072, 3072, 40.0)),
        _wl("mlp", 2, "FLUX.1 MLP fc1 4608x3072->12288, tanh-GELU, fc2 12288->3072, NVFP4 g16",
            LayerShape("fc1", 4608, 3072, 12288, 40.0, layer_id=0),
            LayerShape("fc2", 4608, 12288, 3072, 40.0, outliers=False, layer_id=1)),
        _wl("qkv_int4", 3, "fused QKV projection 4608x3072->9216, INT4 g64",
            LayerShape("qkv", 4608, 3072, 9216, 40.0, fmt="int4")),
        _wl("block_b4", 4, "FLUX.1-dev double-stream block linears at batch 4 (M=18432) + adaLN W4A16 (M=4)",
            LayerShape("qkv", 18432, 3072, 9216, 40.0, layer_id=0),
            LayerShape("out", 18432, 3072, 3072, 40.0, layer_id=1),
            LayerShape("fc1", 18432, 3072, 12288, 40.0, layer_id=2),
            LayerShape("fc2", 18432, 12288, 3072, 40.0, outliers=False, layer_id=3),
            LayerShape("adaln", 4, 3072, 18432, 40.0, fmt="w4a16", outliers=False, layer_id=4)),
    ]
}


def rng(workload_id: int, layer_id: int, role: int) -> np.random.Generator:
    return np.random.default_rng([workload_id, layer_id, role])


def to_bf16(a: np.ndarray) -> np.ndarray:
    """Round to BF16 (nearest even) and return float32 values."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.bfloat16).to(torch.float32).numpy()


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """Raw BF16 bit patterns (uint16) of a float32 array of BF16 values."""
    a32 = np.ascontiguousarray(a, dtype=np.float32)
    bits = a32.view(np.uint32)
    if np.any(bits & 0xFFFF):
        raise ValueError("array holds values that are not BF16-representable")
    return (bits >> 16).astype(np.uint16)


def from_bf16_bits(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint32) << 16).view(np.float32)


def outlier_channels(workload_id: int, layer_id: int, K: int) -> np.ndarray:
    n = int(np.floor(OUTLIER_FRACTION * K))
    g = rng(workload_id, layer_id, ROLE_OUTLIERS)
    return np.sort(g.choice(K, size=n, replace=False))


def activations(workload_id: int, layer_id: int, M: int, K: int, role: int,
                outliers: bool = True) -> np.ndarray:
    """X ~ N(0,1), outlier channels x50, rounded to BF16 (float32 values)."""
    x = rng(workload_id, layer_id, role).standard_normal((M, K))
    if outliers:
        x[:, outlier_channels(workload_id, layer_id, K)] *= OUTLIER_GAIN
    return to_bf16(x)


def correlated_activations(workload_id: int, layer_id: int, M: int, K: int, role: int,
                           latent_rank: int, outliers: bool = True) -> np.ndarray:
    """X = Z A + 0.5 E: every channel mixes the same latent_rank directions
    (Z ~ N(0,1) [M, r] drawn per batch, A ~ N(0, 1/r) [r, K] fixed per layer),
    plus independent N(0,1) noise E; outlier channels x50; rounded to BF16.
    Channels of a real layer's input are correlated like this, and GPTQ's
    error feedback works through exactly that correlation."""
    g = rng(workload_id, layer_id, role)
    A = rng(workload_id, layer_id, ROLE_X_LATENT).standard_normal((latent_rank, K)) / np.sqrt(latent_rank)
    x = g.standard_normal((M, latent_rank)) @ A + LATENT_NOISE * g.standard_normal((M, K))
    if outliers:
        x[:, outlier_channels(workload_id, layer_id, K)] *= OUTLIER_GAIN
    return to_bf16(x)


def weights(workload_id: int, layer_id: int, K: int, N: int, sigma0: float,
            spikes: int = SPIKES) -> np.ndarray:
    """W = N(0, 1/K) + sum_i sigma_i u_i v_i^T, rounded to BF16."""
    w = rng(workload_id, layer_id, ROLE_W_NOISE).standard_normal((K, N)) / np.sqrt(K)
    if spikes:
        u, _ = np.linalg.qr(rng(workload_id, layer_id, ROLE_U).standard_normal((K, spikes)))
        v, _ = np.linalg.qr(rng(workload_id, layer_id, ROLE_V).standard_normal((N, spikes)))
        sig = sigma0 * SPIKE_DECAY ** np.arange(spikes)
        w += (u * sig) @ v.T
    return to_bf16(w)


def bias(workload_id: int, layer_id: int, N: int) -> np.ndarray:
    b = rng(workload_id, layer_id, ROLE_BIAS).standard_normal(N) * np.sqrt(BIAS_VARIANCE)
    return to_bf16(b)


def layer(workload: str, layer_name: Optional[str] = None, M: Optional[int] = None,
          with_run: bool = True, with_heldout: bool = False) -> dict:
    """All seeded inputs of one layer of a workload.

    Returns a dict with ``shape`` (LayerShape), ``W`` [K,N], ``bias`` [N],
    ``Xc`` [256,K] (calibration batch), ``X`` [M,K] (run batch) and
    optionally ``Xh`` (a held-out batch of 256 tokens).  All float32 with
    BF16 values.  ``M`` overrides the run-batch token count.

    For a layer whose input is another layer's output (fc2), only W and bias
    are produced here: its activations come from running the previous layer.
    """
    wl = WORKLOADS[workload]
    shp = wl.layers[0] if layer_name is None else next(l for l in wl.layers if l.name == layer_name)
    M = shp.M if M is None else M
    wid, lid = wl.workload_id, shp.layer_id
    out = {"shape": dataclasses.replace(shp, M=M),
           "W": weights(wid, lid, shp.K, shp.N, shp.sigma0),
           "bias": bias(wid, lid, shp.N)}
    chained = (shp.name == "fc2")
    if not chained:
        out["Xc"] = activations(wid, lid, CALIB_TOKENS, shp.K, ROLE_X_CALIB, shp.outliers)
        if with_run:
            out["X"] = activations(wid, lid, M, shp.K, ROLE_X_RUN, shp.outliers)
        if with_heldout:
            out["Xh"] = activations(wid, lid, CALIB_TOKENS, shp.K, ROLE_X_HELDOUT, shp.outliers)
    return out


def custom_layer(seed: int, M: int, K: int, N: int, sigma0: float = 20.0,
                 outliers: bool = True, calib_tokens: int = CALIB_TOKENS,
                 latent_rank: int = 0, with_heldout: bool = False) -> dict:
    """Same recipe at an arbitrary shape (parity sweeps over tails and sizes).
    latent_rank > 0 draws the activations from ``correlated_activations``."""
    wid, lid = 1000 + seed, 0
    shp = LayerShape(f"custom{seed}", M, K, N, sigma0, outliers=outliers)

    def acts(m, role):
        if latent_rank > 0:
            return correlated_activations(wid, lid, m, K, role, latent_rank, outliers)
        return activations(wid, lid, m, K, role, outliers)

    out = {"shape": shp,
           "W": weights(wid, lid, K, N, sigma0, spikes=min(SPIKES, K, N)),
           "bias": bias(wid, lid, N),
           "Xc": acts(calib_tokens, ROLE_X_CALIB),
           "X": acts(M, ROLE_X_RUN)}
    if with_heldout:
        out["Xh"] = acts(calib_tokens, ROLE_X_HELDOUT)
    return out
