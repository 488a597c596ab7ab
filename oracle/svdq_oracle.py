"""CPU oracle for the SVDQuant W4A4 linear layer -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this module.  The product
(the C-ABI library and its Python binding) never imports, links or calls it,
and this module imports nothing from the product.

Sources (the two pages that describe the method):
  [P] SOTA-314, practice record "SVDQuant" -- sections "Do this",
      "What it buys", "Conditions".
  [N] NOTE-257, note record "SVDQuant" -- sections "Contribution",
      "Key results" (Propositions 4.1/4.2, Eckart-Young, Figure 5, LoRC
      control, the fused-kernel pairings), "Claims" (C1-C4), "Limitations".

The layer computes
    Y = Q(X diag(lam)^-1) Q(R) + (X diag(lam)^-1 L1) L2 + b,
    W_hat = diag(lam) W,  L1 = U Sigma[:, :r],  L2 = V^T[:r, :],
    R = W_hat - L1 L2 quantized to NVFP4 (g16, E4M3 scales) or INT4 (g64, 16-bit scales).
Everything is float64 except where a floating-point decision picks an integer
(a quantization code or a scale byte): those steps run in IEEE float32, the
precision the GPU kernels use, so codes and scales can be compared bit for bit.

Readings where the pages are silent (each listed with its reason in the
design notes of the repository):
  * smoothing: the SmoothQuant form lam_k = max|Xc[:,k]|^a / max|W[k,:]|^(1-a),
    a = 0.5, computed in float32 with IEEE sqrt and division; a channel whose
    activation or weight maximum is zero gets lam = 1;
  * the 1/lam of the down branch is folded into the stored down factor:
    L1d = bf16(diag(1/lam) L1), L2b = bf16(L2);
  * the residual subtracts the 16-bit branch actually stored:
    R = fp32(W_hat - diag(lam) L1d L2b);
  * NVFP4 carries a power-of-two float32 tensor scale per operand:
    g_w = 2^ceil(log2(amax|R| / (6*448))) for the residual and
    g_x = 2^ceil(log2(4 * amax|Xc diag(1/lam)| / (6*448))) for activations
    (fixed from the calibration batch, with 4x headroom);
  * RTN means round to nearest, ties to even, saturating at the format's
    largest finite value; a group whose E4M3 scale rounds to zero gets +0 codes;
  * the code of a group element is E2M1(fp32(v * fp32(1/(s*g)))), with v the
    float32 value fed to the quantizer;
  * INT4 is symmetric in [-7, 7], its 16-bit scale is BF16: s = bf16(fp32(a * fp32(1/7)));
  * two codes per byte, the even k in the low nibble;
  * W8A8 (rank 16 at 8 bits; the pages give no 8-bit group size): INT8
    symmetric in [-127, 127] with one group per row -- per token for the
    activations, per output channel for the residual -- and float32 scales
    s = fp32(a * fp32(1/127)), code = rint_even(fp32(v * fp32(1/s)));
  * GPTQ (the pages' residual quantizer, named but not restated) is the
    published column-by-column algorithm: H = X_hat^T X_hat of the smoothed
    calibration batch, dead channels H_kk = 1, damping 1% of the mean
    diagonal, U = upper Cholesky factor of H^-1, channels in natural order,
    a group's scale fixed from the updated values when the group starts.
"""
from __future__ import annotations

import math
from typing import Dict, Optional

import numpy as np

F32 = np.float32

E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
E4M3_MAX = 448.0
E2M1_MAX = 6.0
NVFP4_GROUP = 16
INT4_GROUP = 64
INT4_QMAX = 7
INT8_QMAX = 127


# --------------------------------------------------------------------------
# Number formats  [P "Do this": "group size 64 with 16-bit scales for INT4,
# group size 16 with FP8 scales for NVFP4"; N "Key results", same sentence]
# --------------------------------------------------------------------------

def _round_to_quantum(x: np.ndarray, quantum: np.ndarray) -> np.ndarray:
    """Round x to the nearest multiple of a power-of-two quantum, ties to even."""
    return np.rint(x / quantum) * quantum


def bf16_round(x) -> np.ndarray:
    """BF16 round-to-nearest-even of the exact value of x (float64 result).

    BF16 keeps 8 significant bits and float32's exponent range (subnormal
    quantum 2^-133)."""
    x = np.asarray(x, dtype=np.float64)
    _, e = np.frexp(x)                       # |x| = m 2^e, m in [0.5, 1)
    q = np.ldexp(1.0, np.maximum(e - 8, -133))
    out = _round_to_quantum(x, q)
    big = np.abs(out) > 3.3895313892515355e38
    return np.where(big, np.copysign(np.inf, x), out)


def fp32(x) -> np.ndarray:
    """IEEE float32 rounding (nearest even)."""
    return np.asarray(x, dtype=np.float64).astype(F32)


def e4m3_round_satfinite(t) -> np.ndarray:
    """Value of E4M3 (bias 7, 3 mantissa bits, max 448, subnormal quantum 2^-9)
    nearest to t >= 0, ties to even, values above 448 clamp to 448."""
    t = np.asarray(t, dtype=np.float64)
    a = np.abs(t)
    _, e = np.frexp(a)
    # normal binade [2^(e-1), 2^e) keeps 4 significant bits: quantum 2^(e-4);
    # below 2^-6 the quantum stays 2^-9 (subnormals).
    q = np.ldexp(1.0, np.maximum(e - 4, -9))
    r = _round_to_quantum(a, q)
    r = np.minimum(r, E4M3_MAX)
    return np.copysign(r, t)


def e4m3_encode(v) -> np.ndarray:
    """Byte of an E4M3-representable non-negative value (sign bit 0)."""
    v = np.asarray(v, dtype=np.float64)
    if np.any(v < 0):
        raise ValueError("scales are non-negative")
    out = np.zeros(v.shape, dtype=np.uint8)
    nz = v > 0
    sub = nz & (v < 2.0 ** -6)
    out[sub] = (v[sub] / 2.0 ** -9).astype(np.uint8)
    nrm = nz & ~sub
    _, e = np.frexp(v[nrm])                  # v = m 2^e, leading bit 2^(e-1)
    ebits = (e - 1) + 7
    mbits = (v[nrm] / np.ldexp(1.0, e - 1) - 1.0) * 8
    out[nrm] = (ebits * 8 + mbits).astype(np.uint8)
    return out


def e4m3_decode(b) -> np.ndarray:
    b = np.asarray(b, dtype=np.int64)
    s = np.where(b & 0x80, -1.0, 1.0)
    e = (b >> 3) & 0xF
    m = b & 0x7
    val = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.ldexp(1.0, e - 7))
    val = np.where((e == 15) & (m == 7), np.nan, val)
    return s * val


def e2m1_encode(q) -> np.ndarray:
    """4-bit E2M1 code of float q: nearest grid value, ties to the even code,
    saturating at 6, sign bit kept (so -0.1 -> 0b1000)."""
    q = np.asarray(q, dtype=np.float64)
    a = np.abs(q)
    # grid midpoints; at a tie the even code (0, 2, 4, 6) wins
    mag = np.select(
        [a <= 0.25, a < 0.75, a <= 1.25, a < 1.75, a <= 2.5, a < 3.5, a <= 5.0],
        [0, 1, 2, 3, 4, 5, 6], default=7).astype(np.uint8)
    sign = np.signbit(q).astype(np.uint8) << 3
    return sign | mag


def e2m1_decode(c) -> np.ndarray:
    c = np.asarray(c, dtype=np.int64)
    return np.where(c & 0x8, -1.0, 1.0) * E2M1_GRID[c & 0x7]


def pack_nibbles(codes: np.ndarray) -> np.ndarray:
    """[rows, K] 4-bit codes -> [rows, K/2] bytes, even k in the low nibble."""
    c = np.asarray(codes, dtype=np.uint8) & 0xF
    return (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)


def unpack_nibbles(packed: np.ndarray) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty((p.shape[0], p.shape[1] * 2), dtype=np.uint8)
    out[:, 0::2] = p & 0xF
    out[:, 1::2] = p >> 4
    return out


def int4_decode(c) -> np.ndarray:
    """Two's-complement 4-bit nibble -> integer."""
    c = np.asarray(c, dtype=np.int64) & 0xF
    return np.where(c >= 8, c - 16, c)


# --------------------------------------------------------------------------
# Group quantizers  [P "Do this": per-group symmetric quantization on both sides]
# --------------------------------------------------------------------------

def pow2_exponent_ceil(x: float) -> int:
    """Smallest integer e with 2^e >= x (x > 0); 0 for x == 0."""
    if x <= 0:
        return 0
    m, e = math.frexp(x)                     # x = m 2^e, m in [0.5, 1)
    return e - 1 if m == 0.5 else e


def nvfp4_group_scale(a: np.ndarray, g_exp: int):
    """Scale of NVFP4 groups with float32 maxima a: t = fp32(a * c) with
    c = fp32(1/6) * 2^-g_exp; s = E4M3(t).  Returns s (float64 holding the E4M3
    value) and inv = fp32(1 / fp32(s * g)), 0 where s == 0."""
    a = np.asarray(a, dtype=F32)
    c = F32(np.ldexp(np.float64(F32(1.0 / 6.0)), -g_exp))
    t = (a * c).astype(F32)                                      # one float32 multiply
    s = e4m3_round_satfinite(t.astype(np.float64))
    sg = fp32(s * np.ldexp(1.0, g_exp))                          # exact (power-of-two scaling)
    with np.errstate(divide="ignore"):
        inv = (F32(1.0) / sg).astype(F32)                        # IEEE float32 division
    return s, np.where(s == 0, F32(0.0), inv).astype(F32)


def nvfp4_codes(v: np.ndarray, s: np.ndarray, inv: np.ndarray) -> np.ndarray:
    """E2M1 codes of float32 values v under scales s / reciprocals inv
    (broadcast against v): code = E2M1(fp32(v * inv)); +0 where s == 0."""
    q = (np.asarray(v, dtype=F32) * inv).astype(F32)             # one float32 multiply
    codes = e2m1_encode(q.astype(np.float64))
    return np.where(s == 0, np.uint8(0), codes).astype(np.uint8)


def nvfp4_quantize(v: np.ndarray, g_exp: int) -> Dict[str, np.ndarray]:
    """NVFP4 quantization of the rows of v (float32, [rows, K]) in groups of 16
    consecutive k, with tensor scale g = 2^g_exp.

    Per group: a = max|v|; t = fp32(a * c) with c = fp32(1/6) * 2^-g_exp;
    s = E4M3(t); s == 0 -> all codes +0; else inv = fp32(1 / (s * g)),
    code = E2M1(fp32(v * inv)).  Returns codes [rows, K] (4-bit), the E4M3
    scale bytes [rows, K/16], scale values and the dequantized values
    E2M1(code) * s * g (float64)."""
    v = np.asarray(v, dtype=F32)
    rows, K = v.shape
    assert K % NVFP4_GROUP == 0
    grp = v.reshape(rows, K // NVFP4_GROUP, NVFP4_GROUP)
    a = np.max(np.abs(grp), axis=2)                              # float32, exact
    s, inv = nvfp4_group_scale(a, g_exp)
    codes = nvfp4_codes(grp, s[:, :, None], inv[:, :, None])
    deq = e2m1_decode(codes) * (s * np.ldexp(1.0, g_exp))[:, :, None]
    return {"codes": codes.reshape(rows, K), "scale_bytes": e4m3_encode(s),
            "scales": s, "deq": deq.reshape(rows, K)}


def int4_group_scale(a: np.ndarray):
    """Scale of INT4 groups with float32 maxima a: s = bf16(fp32(a * fp32(1/7)));
    returns s (float64 holding the BF16 value) and inv = fp32(1 / s), 0 where s == 0."""
    a = np.asarray(a, dtype=F32)
    s = bf16_round((a * F32(1.0 / 7.0)).astype(F32))
    with np.errstate(divide="ignore"):
        inv = (F32(1.0) / s.astype(F32)).astype(F32)
    return s, np.where(s == 0, F32(0.0), inv).astype(F32)


def int4_codes(v: np.ndarray, inv: np.ndarray) -> np.ndarray:
    """code = clamp(rint_even(fp32(v * inv)), -7, 7) as int8 (0 where inv == 0)."""
    q = (np.asarray(v, dtype=F32) * inv).astype(F32)
    return np.clip(np.rint(q.astype(np.float64)), -INT4_QMAX, INT4_QMAX).astype(np.int8)


def int4_quantize(v: np.ndarray) -> Dict[str, np.ndarray]:
    """Symmetric INT4 quantization of the rows of v (float32) in groups of 64.

    Per group: a = max|v|; s = bf16(fp32(a * fp32(1/7))); s == 0 -> codes 0;
    else code = clamp(rint_even(fp32(v * fp32(1/s))), -7, 7).  Returns codes
    [rows, K] as int8, scales [rows, K/64] (float64 BF16 values) and deq."""
    v = np.asarray(v, dtype=F32)
    rows, K = v.shape
    assert K % INT4_GROUP == 0
    grp = v.reshape(rows, K // INT4_GROUP, INT4_GROUP)
    a = np.max(np.abs(grp), axis=2)
    s, inv = int4_group_scale(a)
    codes = int4_codes(grp, inv[:, :, None])
    deq = codes.astype(np.float64) * s[:, :, None]
    return {"codes": codes.reshape(rows, K), "scales": s, "deq": deq.reshape(rows, K)}


def int8_row_scale(a: np.ndarray):
    """Scale of INT8 rows with float32 maxima a: s = fp32(a * fp32(1/127));
    returns s (float32) and inv = fp32(1 / s), 0 where s == 0."""
    a = np.asarray(a, dtype=F32)
    s = (a * F32(1.0 / 127.0)).astype(F32)
    with np.errstate(divide="ignore"):
        inv = (F32(1.0) / s).astype(F32)
    return s, np.where(s == 0, F32(0.0), inv).astype(F32)


def int8_quantize_rows(v: np.ndarray) -> Dict[str, np.ndarray]:
    """Symmetric INT8 quantization of the rows of v (float32, [rows, K]), one
    scale per row: a = max|v|; s = fp32(a * fp32(1/127)); s == 0 -> codes 0;
    else code = clamp(rint_even(fp32(v * fp32(1/s))), -127, 127).  Returns
    codes [rows, K] (int8), scales [rows] (float32 values, as float64) and deq."""
    v = np.asarray(v, dtype=F32)
    a = np.max(np.abs(v), axis=1)
    s, inv = int8_row_scale(a)
    q = (v * inv[:, None]).astype(F32)
    codes = np.clip(np.rint(q.astype(np.float64)), -INT8_QMAX, INT8_QMAX).astype(np.int8)
    s64 = s.astype(np.float64)
    return {"codes": codes, "scales": s64, "deq": codes.astype(np.float64) * s64[:, None]}


def int4_nibbles(codes: np.ndarray) -> np.ndarray:
    return (np.asarray(codes, dtype=np.int64) & 0xF).astype(np.uint8)


# --------------------------------------------------------------------------
# Offline preparation  [P "Do this", first three paragraphs; N "Key results"]
# --------------------------------------------------------------------------

def smoothing_factors(Xc: np.ndarray, W: np.ndarray, alpha: float = 0.5):
    """Per-input-channel smoothing factors lam and 1/lam (float32).

    [P "Do this": smoothing shifts the outliers out of the activations into
    the weights.]  lam_k = max|Xc[:,k]|^alpha / max|W[k,:]|^(1-alpha).  For
    alpha = 0.5 this is fp32(sqrt(ax)) / fp32(sqrt(aw)) in float32; other alphas
    are evaluated in float64 and rounded once."""
    ax = np.max(np.abs(np.asarray(Xc, dtype=F32)), axis=0).astype(F32)
    aw = np.max(np.abs(np.asarray(W, dtype=F32)), axis=1).astype(F32)
    if alpha == 0.5:
        with np.errstate(divide="ignore", invalid="ignore"):
            lam = (np.sqrt(ax) / np.sqrt(aw)).astype(F32)
    else:
        with np.errstate(divide="ignore", invalid="ignore"):
            lam = fp32(np.power(ax.astype(np.float64), alpha)
                       / np.power(aw.astype(np.float64), 1.0 - alpha))
    lam = np.where((ax == 0) | (aw == 0), F32(1.0), lam).astype(F32)
    inv = (F32(1.0) / lam).astype(F32)
    return lam, inv


def svd_split(W_hat: np.ndarray, rank: int):
    """Top-r SVD factors of W_hat = U Sigma V^T: L1 = U[:, :r] Sigma[:r] (K x r),
    L2 = V^T[:r, :] (r x N).  [N "Key results": "L1 = U Sigma_{:,:r},
    L2 = V_{:r,:}" -- read as the top r rows of V^T; the sign of each singular
    pair is free.]  Returns (L1, L2, singular values)."""
    U, S, Vt = np.linalg.svd(np.asarray(W_hat, dtype=np.float64), full_matrices=False)
    L1, L2 = U[:, :rank] * S[:rank], Vt[:rank, :]
    if rank > len(S):
        # a matrix of rank < r: the branch holds all of it, the extra directions are zero
        L1 = np.pad(L1, ((0, 0), (0, rank - len(S))))
        L2 = np.pad(L2, ((0, rank - len(S)), (0, 0)))
    return L1, L2, S


def prepare(W: np.ndarray, bias: Optional[np.ndarray], Xc: np.ndarray, fmt: str = "nvfp4",
            rank: int = 32, alpha: float = 0.5, svd=None, method: str = "rtn",
            gptq_U: Optional[np.ndarray] = None) -> Dict[str, np.ndarray]:
    """Offline pipeline: smooth -> SVD of W_hat -> keep the top r directions in
    16 bits -> quantize only the residual.  [P "Do this": "Compute the SVD of
    the smoothed weight W_hat, keep the top r singular directions in 16 bits,
    and quantize only the residual R = W_hat - L1 L2"; rank 32 at 4 bits.]

    ``svd`` may supply (L1, L2) to replace the LAPACK split (used to compare
    against another implementation's factors on shared inputs).  ``method``
    picks the residual quantizer: "rtn" (round to nearest) or "gptq"; ``gptq_U``
    may supply the GPTQ factor (same purpose as ``svd``)."""
    W = np.asarray(W, dtype=np.float64)
    K, N = W.shape
    lam, inv = smoothing_factors(Xc, W, alpha)
    W_hat = lam.astype(np.float64)[:, None] * W
    if rank > 0:
        if svd is None:
            L1, L2, S = svd_split(W_hat, rank)
        else:
            L1, L2 = svd
            S = None
        L1d = bf16_round(inv.astype(np.float64)[:, None] * L1)
        L2b = bf16_round(L2)
        branch = (lam.astype(np.float64)[:, None] * L1d) @ L2b
    else:
        L1 = np.zeros((K, 0)); L2 = np.zeros((0, N)); S = None
        L1d = np.zeros((K, 0)); L2b = np.zeros((0, N)); branch = 0.0
    R = fp32(W_hat - branch)
    out = {"fmt": fmt, "rank": rank, "alpha": alpha, "K": K, "N": N,
           "lam": lam, "inv_lam": inv, "L1": L1, "L2": L2, "S": S,
           "L1d": L1d, "L2b": L2b, "R": R,
           "bias": np.zeros(N) if bias is None else np.asarray(bias, dtype=np.float64)}
    if method == "rtn":
        out.update(quantize_weights(R, fmt))
    elif method == "gptq":
        U = gptq_factor(gptq_hessian(Xc, inv)) if gptq_U is None else gptq_U
        out.update(gptq_quantize(R, U, fmt))
        out["gptq_U"] = U
    else:
        raise ValueError(method)
    out["g_x_exp"] = activation_tensor_exponent(Xc, inv) if fmt == "nvfp4" else 0
    return out


def attach_lora(prep: Dict[str, np.ndarray], A: np.ndarray, B: np.ndarray, scale: float) -> Dict[str, np.ndarray]:
    """A LoRA adapter W -> W + scale A B concatenated into the 16-bit branch
    without re-quantizing anything [P "Known implementations": the paper's
    engine loads off-the-shelf LoRA adapters without re-quantization]:
        L1d' = [L1d | bf16(A)],  L2b' = [L2b ; bf16(fp32(scale) B)],
    rank 32 + r; lam, the residual and its codes and scales are unchanged.  A
    acts on the unsmoothed input, like L1d (which carries 1/lam)."""
    A = bf16_round(np.asarray(A, dtype=np.float64))
    Bs = bf16_round(bf16_round(np.asarray(B, dtype=np.float64)) * float(np.float32(scale)))
    out = dict(prep)
    out["L1d"] = np.hstack([np.asarray(prep["L1d"], dtype=np.float64).reshape(prep["K"], -1), A])
    out["L2b"] = np.vstack([np.asarray(prep["L2b"], dtype=np.float64).reshape(-1, prep["N"]), Bs])
    out["rank"] = out["L1d"].shape[1]
    out["lora_r"] = A.shape[1]
    return out


def weight_tensor_exponent(R: np.ndarray) -> int:
    """g_w = 2^ceil(log2(amax|R| / (6 * 448)))."""
    return pow2_exponent_ceil(float(np.max(np.abs(R))) / (E2M1_MAX * E4M3_MAX))


def activation_tensor_exponent(Xc: np.ndarray, inv_lam: np.ndarray) -> int:
    """g_x = 2^ceil(log2(4 * amax|fp32(Xc * inv_lam)| / (6 * 448)))."""
    v = (np.asarray(Xc, dtype=F32) * inv_lam[None, :]).astype(F32)
    return pow2_exponent_ceil(4.0 * float(np.max(np.abs(v))) / (E2M1_MAX * E4M3_MAX))


def quantize_weights(R: np.ndarray, fmt: str, g_exp: Optional[int] = None) -> Dict[str, np.ndarray]:
    """Quantize the residual R [K, N] column by column: groups run along K for
    each output n, so codes are [N, K] (K-major)."""
    Rt = np.ascontiguousarray(np.asarray(R, dtype=F32).T)
    if fmt == "nvfp4":
        e = weight_tensor_exponent(Rt) if g_exp is None else g_exp
        q = nvfp4_quantize(Rt, e)
        return {"g_w_exp": e, "w_codes": q["codes"], "w_scale_bytes": q["scale_bytes"],
                "w_scales": q["scales"], "w_deq": q["deq"]}
    if fmt in ("int4", "w4a16"):
        q = int4_quantize(Rt)
        return {"g_w_exp": 0, "w_codes": q["codes"], "w_scales": q["scales"], "w_deq": q["deq"]}
    if fmt == "w8a8":
        q = int8_quantize_rows(Rt)                    # one scale per output channel
        return {"g_w_exp": 0, "w_codes": q["codes"], "w_scales": q["scales"], "w_deq": q["deq"]}
    raise ValueError(fmt)


# --------------------------------------------------------------------------
# GPTQ residual quantization  [P "Do this": the residual is quantized with
# GPTQ rather than round-to-nearest; N "Key results", the quality table rows]
#
# The pages name GPTQ without restating it; this is the published algorithm
# (Frantar et al., "GPTQ: Accurate Post-Training Quantization for Generative
# Pre-trained Transformers", 2022) in its plain column-by-column form: the
# lazy block updates of that paper only reorder the same arithmetic.
#   * the loss of output column n is ||X_hat (r_n - q_n)||^2 with X_hat the
#     smoothed calibration activations, so H = X_hat^T X_hat for every n;
#   * a channel that never fires (H_kk = 0) gets H_kk = 1, then every H_kk
#     grows by 1% of the mean diagonal (the paper's damping);
#   * U = upper Cholesky factor of H^-1 (H^-1 = U^T U);
#   * input channels k are visited in order; when k starts a group, that
#     group's scale is fixed from the current (already updated) values;
#     w_k is quantized with it, err = (w_k - deq_k) / U_kk and every later
#     channel j > k moves by -U_kj err.
# Working values are float64; the quantizer sees their float32 rounding and
# takes its decisions exactly as round-to-nearest does.
# --------------------------------------------------------------------------

GPTQ_DAMP = 0.01


def gptq_hessian(Xc: np.ndarray, inv_lam: np.ndarray, damp: float = GPTQ_DAMP) -> np.ndarray:
    """Damped H = X_hat^T X_hat (float64), X_hat = fp32(Xc * inv_lam)."""
    Xh = smoothed_activations(Xc, inv_lam).astype(np.float64)
    H = Xh.T @ Xh
    d = np.diag(H).copy()
    dead = np.flatnonzero(d == 0)
    H[dead, dead] = 1.0
    H[np.diag_indices_from(H)] += damp * float(np.mean(np.diag(H)))
    return H


def gptq_factor(H: np.ndarray) -> np.ndarray:
    """Upper-triangular U with positive diagonal and U^T U = H^-1."""
    Hinv = np.linalg.inv(np.asarray(H, dtype=np.float64))
    Hinv = 0.5 * (Hinv + Hinv.T)
    return np.linalg.cholesky(Hinv).T


def gptq_quantize(R: np.ndarray, U: np.ndarray, fmt: str, g_exp: Optional[int] = None) -> Dict[str, np.ndarray]:
    """GPTQ quantization of the residual R [K, N] with factor U [K, K]; the
    result has the keys of quantize_weights (codes [N, K], K-major).  For NVFP4
    the tensor scale g_w comes from the unmodified R, as round-to-nearest's does."""
    W = np.array(R, dtype=F32).astype(np.float64)
    K, N = W.shape
    U = np.asarray(U, dtype=np.float64)
    if fmt == "nvfp4":
        G = NVFP4_GROUP
        e = weight_tensor_exponent(R) if g_exp is None else g_exp
        g = np.ldexp(1.0, e)
    elif fmt in ("int4", "w4a16"):
        G = INT4_GROUP
        e = 0
    else:
        raise ValueError(fmt)
    codes = np.zeros((N, K), dtype=np.uint8 if fmt == "nvfp4" else np.int8)
    scales = np.zeros((N, K // G))
    deq = np.zeros((N, K))
    fed = np.zeros((N, K))                  # the working value of w_k when it is quantized
    for k in range(K):
        if k % G == 0:
            a = np.max(np.abs(W[k:k + G, :].astype(F32)), axis=0)
            s, inv = nvfp4_group_scale(a, e) if fmt == "nvfp4" else int4_group_scale(a)
            scales[:, k // G] = s
        fed[:, k] = W[k, :]
        v = W[k, :].astype(F32)
        if fmt == "nvfp4":
            c = nvfp4_codes(v, s, inv)
            d = e2m1_decode(c) * (s * g)
        else:
            c = int4_codes(v, inv)
            d = c.astype(np.float64) * s
        codes[:, k] = c
        deq[:, k] = d
        err = (W[k, :] - d) / U[k, k]
        W[k + 1:, :] -= np.outer(U[k, k + 1:], err)
    out = {"g_w_exp": e, "w_codes": codes, "w_scales": scales, "w_deq": deq, "w_fed": fed}
    if fmt == "nvfp4":
        out["w_scale_bytes"] = e4m3_encode(scales)
    return out


def smoothed_activations(X: np.ndarray, inv_lam: np.ndarray) -> np.ndarray:
    """x_hat = fp32(x * inv_lam): one IEEE float32 multiply per element."""
    return (np.asarray(X, dtype=F32) * np.asarray(inv_lam, dtype=F32)[None, :]).astype(F32)


def quantize_activations(X: np.ndarray, inv_lam: np.ndarray, fmt: str, g_x_exp: int = 0):
    """Q(X diag(lam)^-1), per token in groups along K (W8A8: one group per token)."""
    v = smoothed_activations(X, inv_lam)
    if fmt == "nvfp4":
        return nvfp4_quantize(v, g_x_exp)
    if fmt == "w8a8":
        return int8_quantize_rows(v)
    return int4_quantize(v)


def down_projection(X: np.ndarray, L1d: np.ndarray) -> np.ndarray:
    """XL = bf16(X L1d), accumulated in float64.  With 1/lam folded into L1d
    this is (X diag(lam)^-1) L1, the branch's down projection [N "Key
    results": "Down Projection with Quantize (shared input)"]."""
    return bf16_round(np.asarray(X, dtype=np.float64) @ np.asarray(L1d, dtype=np.float64))


def gelu_tanh(y: np.ndarray) -> np.ndarray:
    """tanh approximation of GELU: 0.5 y (1 + tanh(u)), u = sqrt(2/pi) (y + 0.044715 y^3).

    Evaluated as y / (1 + exp(-2u)), the same function (0.5 (1 + tanh u) is the
    logistic function of 2u) without the cancellation of 1 + tanh(u) for u << 0,
    which loses every digit below y = -5.6 in float64."""
    y = np.asarray(y, dtype=np.float64)
    u = math.sqrt(2.0 / math.pi) * (y + 0.044715 * y ** 3)
    with np.errstate(over="ignore"):
        return y / (1.0 + np.exp(-2.0 * u))


def forward(prep: Dict[str, np.ndarray], X: np.ndarray, gelu: bool = False,
            xq: Optional[Dict[str, np.ndarray]] = None, XL: Optional[np.ndarray] = None):
    """Y = Q(X diag(lam)^-1) Q(R) + (X diag(lam)^-1 L1) L2 + b  (float64), and its
    BF16 rounding (after tanh-GELU when ``gelu``).  [N "Key results":
    "Up Projection with the 4-bit compute (shared output)".]

    ``xq`` / ``XL`` may supply the activation quantization and down projection
    (to evaluate the output on another implementation's intermediate values)."""
    if xq is None:
        xq = quantize_activations(X, prep["inv_lam"], prep["fmt"], prep["g_x_exp"])
    if XL is None:
        XL = down_projection(X, prep["L1d"]) if prep["rank"] > 0 else None
    Y = xq["deq"] @ prep["w_deq"].T
    if prep["rank"] > 0:
        Y = Y + XL @ prep["L2b"]
    Y = Y + prep["bias"][None, :]
    out = gelu_tanh(Y) if gelu else Y
    return {"Y": Y, "Y_act": out, "Y_bf16": bf16_round(out), "XL": XL, "xq": xq}


def w4a16_prepare(W: np.ndarray, bias: Optional[np.ndarray]) -> Dict[str, np.ndarray]:
    """Weight-only INT4 g64 (BF16 scales) for the adaptive-normalization linears
    [P "Do this": "For FLUX.1 the linear layers inside adaptive normalization
    stay W4A16"]: no smoothing, no low-rank branch."""
    W = np.asarray(W, dtype=np.float64)
    q = int4_quantize(np.ascontiguousarray(W.T).astype(F32))
    return {"w_codes": q["codes"], "w_scales": q["scales"], "w_deq": q["deq"],
            "bias": np.zeros(W.shape[1]) if bias is None else np.asarray(bias, dtype=np.float64)}


def w4a16_forward(prep, X: np.ndarray):
    Y = np.asarray(X, dtype=np.float64) @ prep["w_deq"].T + prep["bias"][None, :]
    return {"Y": Y, "Y_bf16": bf16_round(Y)}


# --------------------------------------------------------------------------
# Ablation  [P "Do this"; N "Key results": "naive quantization and SVD-only both
# poor, smoothing alone slightly better, LoRC suboptimal, decompose-then-
# quantize much better, and adding smoothing on top better again"]
# --------------------------------------------------------------------------

def _fake_quant(v: np.ndarray, fmt: str, g_exp: Optional[int] = None, along_rows=True):
    """Dequantized per-row group quantization (NVFP4 with an amax-derived tensor scale)."""
    v = np.asarray(v, dtype=F32)
    if fmt == "nvfp4":
        e = pow2_exponent_ceil(float(np.max(np.abs(v))) / (E2M1_MAX * E4M3_MAX)) if g_exp is None else g_exp
        return nvfp4_quantize(v, e)["deq"]
    return int4_quantize(v)["deq"]


def _qw(W: np.ndarray, fmt: str) -> np.ndarray:
    """Dequantized weight, groups along K (quantize W^T by rows)."""
    return _fake_quant(np.ascontiguousarray(np.asarray(W).T), fmt).T


def _qx(X: np.ndarray, fmt: str, calib: np.ndarray) -> np.ndarray:
    e = pow2_exponent_ceil(4.0 * float(np.max(np.abs(calib))) / (E2M1_MAX * E4M3_MAX))
    return _fake_quant(np.asarray(X, dtype=F32), fmt, e if fmt == "nvfp4" else None)


def _top_r(M: np.ndarray, r: int) -> np.ndarray:
    L1, L2, _ = svd_split(M, r)
    return L1 @ L2


def ablation_errors(W, b, Xc, Xh, rank: int = 32, fmt: str = "nvfp4", alpha: float = 0.5):
    """Relative Frobenius error of each variant's output against the float64
    product Xh W + b, on a held-out batch Xh (not the calibration batch).

    Variants: naive Q(X)Q(W); svd_only X L1 L2 (low-rank part alone);
    smooth Q(X^)Q(W^); lorc Q(X)Q(W) + X E_r with E_r the top-r SVD of W - Q(W);
    dtq Q(X)Q(W - L1L2) + X L1L2; lorc_smooth; svdquant = dtq on the smoothed pair."""
    W = np.asarray(W, dtype=np.float64); Xh64 = np.asarray(Xh, dtype=np.float64)
    b = np.zeros(W.shape[1]) if b is None else np.asarray(b, dtype=np.float64)
    ref = Xh64 @ W + b
    nref = np.linalg.norm(ref)

    def err(Y):
        return float(np.linalg.norm(Y + b - ref) / nref)

    lam, inv = smoothing_factors(Xc, W, alpha)
    Xs = smoothed_activations(Xh, inv).astype(np.float64)
    Xcs = smoothed_activations(Xc, inv)
    Ws = lam.astype(np.float64)[:, None] * W

    out = {}
    qx, qw = _qx(Xh, fmt, Xc), _qw(W, fmt)
    out["naive"] = err(qx @ qw)
    out["svd_only"] = err(Xh64 @ _top_r(W, rank))
    qxs, qws = _qx(Xs, fmt, Xcs), _qw(Ws, fmt)
    out["smooth"] = err(qxs @ qws)
    out["lorc"] = err(qx @ qw + Xh64 @ _top_r(W - qw, rank))
    low = _top_r(W, rank)
    out["dtq"] = err(qx @ _qw(W - low, fmt) + Xh64 @ low)
    out["lorc_smooth"] = err(qxs @ qws + Xs @ _top_r(Ws - qws, rank))
    lows = _top_r(Ws, rank)
    out["svdquant"] = err(qxs @ _qw(Ws - lows, fmt) + Xs @ lows)
    return out
