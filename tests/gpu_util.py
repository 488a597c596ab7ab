"""Helpers for the GPU parity tests: run the library through its C ABI on
torch-owned device buffers and build the oracle's view of the same prepared
layer (shared prepared tensors)."""
import numpy as np

import synthetic as syn
from oracle import svdq_oracle as o

import w4a4_diffusion_transformer_b200 as lib

# Float tolerances of the BF16 output against the oracle's BF16-rounded output.
REL_FRO = 2e-3
MAX_ABS_FRAC = 1e-2


def torch_bf16(x: np.ndarray, device="cuda"):
    import torch
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16).to(device)


def to_numpy_f32(t) -> np.ndarray:
    import torch
    return t.detach().to(torch.float32).cpu().numpy()


def prepare_gpu(d, fmt="nvfp4", rank=32):
    return lib.Layer.prepare(syn.bf16_bits(d["W"]), syn.bf16_bits(d["bias"]),
                             None if fmt == "w4a16" else syn.bf16_bits(d["Xc"]),
                             fmt=fmt, rank=rank, device=0)


def oracle_prep_from(L, gptq_U=None) -> dict:
    """The oracle's prepared layer built from the library's exported tensors
    (residual quantized by GPTQ with factor ``gptq_U`` when one is given)."""
    info = L.info
    r = info["rank"]
    fmt = {lib.INT4: "int4", lib.W8A8_INT8: "w8a8"}.get(info["format"], "nvfp4")
    p = {"fmt": fmt, "rank": r, "K": info["K"], "N": info["N"],
         "lam": L.export("lambda"), "inv_lam": L.export("inv_lambda"),
         "L1d": syn.from_bf16_bits(L.export("L1d")).astype(np.float64) if r else np.zeros((info["K"], 0)),
         "L2b": syn.from_bf16_bits(L.export("L2b")).astype(np.float64) if r else np.zeros((0, info["N"])),
         "bias": L.export("bias").astype(np.float64), "g_x_exp": info["g_x_exp"]}
    if gptq_U is None:
        p.update(o.quantize_weights(L.export("R"), fmt))
    else:
        p.update(o.gptq_quantize(L.export("R"), gptq_U, fmt))
    if lib.load().svdq_tensor_bytes(L._h, lib.TENSORS["lora_A"][0]):
        # an attached LoRA adapter: its stored factors (bf16(scale B) already scaled)
        p = o.attach_lora(p, syn.from_bf16_bits(L.export("lora_A")), syn.from_bf16_bits(L.export("lora_B")), 1.0)
    assert p["g_w_exp"] == info["g_w_exp"]
    return p


def xl_width(L) -> int:
    """Columns of XL: 64 with a LoRA adapter attached (X A in columns 32..63), else 32."""
    return 64 if lib.load().svdq_tensor_bytes(L._h, lib.TENSORS["lora_A"][0]) else 32


def run_quantize(L, X: np.ndarray, mode=0):
    import torch
    M, K = X.shape
    x = torch_bf16(X)
    codes = torch.full((L.act_code_bytes(M),), 0xAB, dtype=torch.uint8, device="cuda")
    scales = torch.full((L.act_scale_bytes(M),), 0xCD, dtype=torch.uint8, device="cuda")
    xl = torch.full((M, xl_width(L)), float("nan"), dtype=torch.bfloat16, device="cuda")
    L.quantize_act(x, M, codes, scales, xl, torch.cuda.current_stream(), mode)
    torch.cuda.synchronize()
    return {"codes": L.act_codes_to_logical(codes.cpu().numpy(), M), "scales_dev": scales.cpu().numpy(),
            "scales": L.act_scales_to_logical(scales.cpu().numpy(), M), "xl": to_numpy_f32(xl),
            "_t": (x, codes, scales, xl)}


def run_forward(L, X: np.ndarray, flags=0, check=True):
    import torch
    M, K = X.shape
    N = L.info["N"]
    x = torch_bf16(X)
    y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    wsb = L.workspace_bytes(M)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    L.forward(x, M, y, ws, wsb, torch.cuda.current_stream(), flags | (lib.FWD_CHECK if check else 0))
    torch.cuda.synchronize()
    return to_numpy_f32(y)


def assert_close_bf16(y: np.ndarray, ref: np.ndarray, what=""):
    assert np.all(np.isfinite(y)), f"{what}: non-finite output"
    err = np.linalg.norm(y.astype(np.float64) - ref) / max(np.linalg.norm(ref), 1e-300)
    mx = np.max(np.abs(y.astype(np.float64) - ref))
    assert err <= REL_FRO, f"{what}: relative Frobenius error {err:.3e} > {REL_FRO}"
    assert mx <= MAX_ABS_FRAC * np.max(np.abs(ref)), f"{what}: max abs error {mx:.3e}"
    return err, mx


def unit_smoothing_layer(seed, K, N, rng=None):
    """A layer whose smoothing factors are exactly 1: the calibration batch's
    column maxima equal the weight's row maxima, so the quantizer sees X itself
    and hand-placed values hit exact E2M1 / E4M3 ties."""
    d = syn.custom_layer(seed, M=8, K=K, N=N, sigma0=5.0, outliers=False, calib_tokens=16)
    aw = np.max(np.abs(d["W"]), axis=1)
    Xc = d["Xc"].copy()
    Xc = np.clip(Xc, -0.5 * aw, 0.5 * aw)
    Xc = syn.to_bf16(Xc)
    Xc[0] = aw
    d["Xc"] = Xc
    return d
