"""SVDQuant W4A4 linear layer for NVIDIA B200 (sm_100a).

A thin ctypes binding over the C ABI in ``include/svdq.h`` (``libsvdq.so``,
built in-tree by ``w4a4_diffusion_transformer_b200.build``).  The binding only
marshals arguments: every step of the layer runs in the library (host C++ for
the offline preparation, CUDA kernels for the forward).  There is no fallback:
if the library is missing, importing ``lib`` raises.

Device memory and streams come from the caller (for example PyTorch tensors:
anything with ``data_ptr()``, or raw integer addresses).  PyTorch tensors and
NumPy arrays are checked before the call: a device operand must be a
contiguous CUDA tensor, a host operand host memory, and each must hold at
least the bytes the call reads or writes (``ValueError`` otherwise).  Raw
addresses and other objects are passed through unchecked.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsvdq.so")

# status codes (svdq_status)
OK, EINVAL, EUNSUPPORTED, ENOMEM, ECUDA, ENOCONVERGE, ETIMEOUT, ESTATE = range(8)
# formats (svdq_format)
NVFP4, INT4, W4A16_INT4, W8A8_INT8 = 0, 1, 2, 3
FORMATS = {"nvfp4": NVFP4, "int4": INT4, "w4a16": W4A16_INT4, "w8a8": W8A8_INT8}
# forward flags
FWD_GELU, FWD_UNFUSED, FWD_NO_BRANCH, FWD_CHECK = 0x1, 0x2, 0x4, 0x8
# exportable tensors (svdq_tensor)
TENSORS = {
    "lambda": (0, np.float32), "inv_lambda": (1, np.float32), "L1": (2, np.float64), "L2": (3, np.float64),
    "L1d": (4, np.uint16), "L2b": (5, np.uint16), "R": (6, np.float32), "sigma": (7, np.float64),
    "w_codes": (8, np.uint8), "w_scales": (9, None), "bias": (10, np.float32), "gptq_U": (11, np.float64),
    "lora_A": (12, np.uint16), "lora_B": (13, np.uint16),
}
# preparation flags (svdq_config.flags)
PREP_GPTQ, PREP_KEEP_GPTQ_FACTOR = 0x1, 0x2

EXPORTED = [
    "svdq_prepare", "svdq_destroy", "svdq_get_info", "svdq_tensor_bytes", "svdq_export",
    "svdq_status_string", "svdq_workspace_bytes", "svdq_linear_forward", "svdq_quantize_act",
    "svdq_gemm", "svdq_act_scale_bytes", "svdq_act_scales_to_logical", "svdq_check",
    "svdq_linear_forward_static", "svdq_act_code_bytes", "svdq_act_codes_to_logical",
    "svdq_selftest_wait_timeout", "svdq_mlp_workspace_bytes", "svdq_mlp_fc1", "svdq_mlp_forward",
    "svdq_set_lora", "svdq_serialized_bytes", "svdq_serialize", "svdq_deserialize",
]
STATIC_WORKSPACE_BYTES = 16 << 20   # SVDQ_STATIC_WORKSPACE_BYTES


class SvdqError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})")


class Config(ctypes.Structure):
    _fields_ = [("format", ctypes.c_int), ("rank", ctypes.c_int), ("alpha", ctypes.c_float),
                ("flags", ctypes.c_uint)]


class LayerInfo(ctypes.Structure):
    _fields_ = [("K", ctypes.c_int), ("N", ctypes.c_int), ("rank", ctypes.c_int), ("format", ctypes.c_int),
                ("device", ctypes.c_int), ("g_x_exp", ctypes.c_int), ("g_w_exp", ctypes.c_int),
                ("svd_iterations", ctypes.c_int), ("svd_tail_energy", ctypes.c_double)]


_lib: Optional[ctypes.CDLL] = None


def load() -> ctypes.CDLL:
    """Load libsvdq.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m w4a4_diffusion_transformer_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, I, SZ, U = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_uint
    sig = {
        "svdq_prepare": (I, [ctypes.POINTER(Config), I, I, P, P, P, I, I, ctypes.POINTER(P)]),
        "svdq_destroy": (None, [P]),
        "svdq_get_info": (I, [P, ctypes.POINTER(LayerInfo)]),
        "svdq_tensor_bytes": (SZ, [P, I]),
        "svdq_export": (I, [P, I, P, SZ]),
        "svdq_status_string": (ctypes.c_char_p, [I]),
        "svdq_workspace_bytes": (SZ, [P, I]),
        "svdq_linear_forward": (I, [P, P, I, P, P, SZ, P, U]),
        "svdq_quantize_act": (I, [P, P, I, P, P, P, P, I]),
        "svdq_gemm": (I, [P, P, P, P, I, P, P, U]),
        "svdq_act_scale_bytes": (SZ, [P, I]),
        "svdq_act_scales_to_logical": (I, [P, P, I, P]),
        "svdq_check": (I, [P, P]),
        "svdq_linear_forward_static": (I, [P, P, I, P, P, U]),
        "svdq_act_code_bytes": (SZ, [P, I]),
        "svdq_act_codes_to_logical": (I, [P, P, I, P]),
        "svdq_selftest_wait_timeout": (I, [P, U, P]),
        "svdq_mlp_workspace_bytes": (SZ, [P, P, I, U]),
        "svdq_mlp_fc1": (I, [P, P, P, I, P, P, P, P, SZ, P, U]),
        "svdq_mlp_forward": (I, [P, P, P, I, P, P, SZ, P, U]),
        "svdq_set_lora": (I, [P, I, P, P, ctypes.c_float]),
        "svdq_serialized_bytes": (SZ, [P]),
        "svdq_serialize": (I, [P, P, SZ]),
        "svdq_deserialize": (I, [P, SZ, I, ctypes.POINTER(P)]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    _lib = L
    return L


def status_string(s: int) -> str:
    return load().svdq_status_string(int(s)).decode()


def _ptr(x) -> Optional[int]:
    """Device/host address of a tensor-like object (data_ptr()), an int, or None."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if hasattr(x, "data_ptr"):
        return int(x.data_ptr())
    if isinstance(x, np.ndarray):
        return int(x.ctypes.data)
    raise TypeError(f"cannot take the address of {type(x)}")


def _held_bytes(x, what: str, device: bool) -> Optional[int]:
    """Bytes held by a tensor or array argument after checking where it lives
    and that it is contiguous; None for raw addresses and unknown objects."""
    if x is None or isinstance(x, int):
        return None
    if isinstance(x, np.ndarray):
        if device:
            raise ValueError(f"{what}: a NumPy array is host memory; this operand is a device buffer")
        if not x.flags.c_contiguous:
            raise ValueError(f"{what}: not contiguous")
        return int(x.nbytes)
    if hasattr(x, "is_cuda") and hasattr(x, "numel"):
        if bool(x.is_cuda) != device:
            raise ValueError(f"{what}: must be a {'CUDA' if device else 'host'} tensor")
        if not x.is_contiguous():
            raise ValueError(f"{what}: not contiguous")
        return int(x.numel()) * int(x.element_size())
    return None


def _need(x, nbytes: int, what: str, device: bool = True):
    have = _held_bytes(x, what, device)
    if have is not None and have < nbytes:
        raise ValueError(f"{what}: holds {have} bytes, the call accesses {nbytes}")


def _stream(s) -> Optional[int]:
    if s is None:
        return None
    if isinstance(s, int):
        return s
    return int(getattr(s, "cuda_stream"))


def _check(status: int, what: str):
    if status != OK:
        raise SvdqError(status, what)


class Layer:
    """A prepared SVDQuant layer (owns its device buffers)."""

    def __init__(self, handle: int):
        self._h = ctypes.c_void_p(handle)
        info = self.info
        self._K, self._N = info["K"], info["N"]
        self._xl_cols = self._xl_width()

    def _xl_width(self) -> int:
        # XL is [M][32] BF16 (zeros past the rank); [M][64] with a LoRA adapter
        return 64 if load().svdq_tensor_bytes(self._h, TENSORS["lora_A"][0]) else 32

    @classmethod
    def prepare(cls, W_bits: np.ndarray, bias_bits: Optional[np.ndarray], calib_bits: Optional[np.ndarray],
                fmt: str = "nvfp4", rank: int = 32, alpha: float = 0.5, device: int = 0,
                flags: int = 0) -> "Layer":
        """W_bits: uint16 [K][N] BF16 bit patterns (Y = X W + b); bias_bits: uint16 [N] or None;
        calib_bits: uint16 [M_calib][K] or None (W4A16); flags: PREP_* bits."""
        L = load()
        W = np.ascontiguousarray(W_bits, dtype=np.uint16)
        if W.ndim != 2:
            raise ValueError(f"W_bits must be [K][N], got shape {W.shape}")
        K, N = W.shape
        b = None if bias_bits is None else np.ascontiguousarray(bias_bits, dtype=np.uint16)
        c = None if calib_bits is None else np.ascontiguousarray(calib_bits, dtype=np.uint16)
        if b is not None and b.size != N:
            raise ValueError(f"bias_bits must hold N = {N} values, got shape {b.shape}")
        if c is not None and (c.ndim != 2 or c.shape[1] != K):
            raise ValueError(f"calib_bits must be [M_calib][K = {K}], got shape {c.shape}")
        cfg = Config(FORMATS[fmt], rank, alpha, flags)
        out = ctypes.c_void_p()
        st = L.svdq_prepare(ctypes.byref(cfg), K, N, _ptr(W), _ptr(b), _ptr(c),
                            0 if c is None else c.shape[0], device, ctypes.byref(out))
        _check(st, "svdq_prepare")
        return cls(out.value)

    def serialize(self) -> bytes:
        """The prepared layer as bytes (svdq_serialize)."""
        n = int(load().svdq_serialized_bytes(self._h))
        buf = np.empty(n, dtype=np.uint8)
        _check(load().svdq_serialize(self._h, _ptr(buf), n), "svdq_serialize")
        return buf.tobytes()

    @classmethod
    def deserialize(cls, data: bytes, device: int = 0) -> "Layer":
        """Rebuild a layer from serialize()'s bytes (svdq_deserialize)."""
        buf = np.frombuffer(data, dtype=np.uint8)
        out = ctypes.c_void_p()
        _check(load().svdq_deserialize(_ptr(buf), buf.size, device, ctypes.byref(out)), "svdq_deserialize")
        return cls(out.value)

    def close(self):
        if self._h is not None and self._h.value:
            load().svdq_destroy(self._h)
        self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self) -> "Layer":
        return self

    def __exit__(self, *exc):
        self.close()
        return False

    @property
    def info(self) -> dict:
        i = LayerInfo()
        _check(load().svdq_get_info(self._h, ctypes.byref(i)), "svdq_get_info")
        return {f: getattr(i, f) for f, _ in LayerInfo._fields_}

    def export(self, name: str) -> np.ndarray:
        tid, dt = TENSORS[name]
        info = self.info
        K, N, r = info["K"], info["N"], info["rank"]
        if dt is None:
            dt = {NVFP4: np.uint8, W8A8_INT8: np.float32}.get(info["format"], np.uint16)
        nbytes = load().svdq_tensor_bytes(self._h, tid)
        buf = np.empty(nbytes // np.dtype(dt).itemsize, dtype=dt)
        _check(load().svdq_export(self._h, tid, _ptr(buf), nbytes), f"svdq_export({name})")
        w8 = info["format"] == W8A8_INT8
        shapes = {"lambda": (K,), "inv_lambda": (K,), "L1": (K, r), "L2": (r, N), "L1d": (K, r),
                  "L2b": (r, N), "R": (K, N), "sigma": (r,), "w_codes": (N, K if w8 else K // 2), "bias": (N,),
                  "w_scales": (N,) if w8 else (N, -1), "gptq_U": (K, K), "lora_A": (K, -1), "lora_B": (-1, N)}
        return buf.reshape(shapes[name])

    def set_lora(self, A_bits: Optional[np.ndarray], B_bits: Optional[np.ndarray], scale: float = 1.0):
        """Attach a LoRA adapter W -> W + scale A B (A_bits uint16 [K][r], B_bits
        uint16 [r][N], BF16 patterns) to the low-rank branch; None removes it."""
        if A_bits is None:
            try:
                _check(load().svdq_set_lora(self._h, 0, None, None, 0.0), "svdq_set_lora")
            finally:
                self._xl_cols = self._xl_width()
            return
        A = np.ascontiguousarray(A_bits, dtype=np.uint16)
        B = np.ascontiguousarray(B_bits, dtype=np.uint16)
        if A.ndim != 2 or B.ndim != 2 or A.shape[0] != self._K or B.shape != (A.shape[1], self._N):
            raise ValueError(f"A is [K = {self._K}][r] and B is [r][N = {self._N}]; got {A.shape} and {B.shape}")
        r = A.shape[1]
        try:
            _check(load().svdq_set_lora(self._h, r, _ptr(A), _ptr(B), float(scale)), "svdq_set_lora")
        finally:
            self._xl_cols = self._xl_width()

    def workspace_bytes(self, M: int) -> int:
        return int(load().svdq_workspace_bytes(self._h, M))

    def act_scale_bytes(self, M: int) -> int:
        return int(load().svdq_act_scale_bytes(self._h, M))

    def act_code_bytes(self, M: int) -> int:
        return int(load().svdq_act_code_bytes(self._h, M))

    def act_codes_to_logical(self, device_layout: np.ndarray, M: int) -> np.ndarray:
        """Activation codes in the GEMM's layout -> uint8 [M][K/2] (two codes per
        byte); W8A8: int8 [M][K]."""
        info = self.info
        if info["format"] == W8A8_INT8:
            out = np.empty((M, info["K"]), dtype=np.int8)
        else:
            out = np.empty((M, info["K"] // 2), dtype=np.uint8)
        src = np.ascontiguousarray(device_layout, dtype=np.uint8)
        _need(src, self.act_code_bytes(M), "device_layout", device=False)
        _check(load().svdq_act_codes_to_logical(self._h, _ptr(src), M, _ptr(out)), "svdq_act_codes_to_logical")
        return out

    def _need_act(self, M: int, X=None, Y=None, codes=None, scales=None, xl=None):
        if M <= 0:
            return                     # the library answers M <= 0 itself
        if X is not None:
            _need(X, M * self._K * 2, "X")
        if Y is not None:
            _need(Y, M * self._N * 2, "Y")
        if codes is not None:
            _need(codes, self.act_code_bytes(M), "codes")
        if scales is not None:
            _need(scales, self.act_scale_bytes(M), "scales")
        if xl is not None:
            _need(xl, M * self._xl_cols * 2, "xl")

    def forward(self, X, M: int, Y, workspace, workspace_bytes: int, stream=None, flags: int = 0):
        self._need_act(M, X=X, Y=Y)
        _need(workspace, workspace_bytes, "workspace")
        _check(load().svdq_linear_forward(self._h, _ptr(X), M, _ptr(Y), _ptr(workspace), workspace_bytes,
                                          _stream(stream), flags), "svdq_linear_forward")

    def forward_static(self, X, M: int, Y, stream=None, flags: int = 0):
        """Forward with the library's built-in device workspace (no caller workspace,
        no allocation); see svdq_linear_forward_static in include/svdq.h."""
        self._need_act(M, X=X, Y=Y)
        _check(load().svdq_linear_forward_static(self._h, _ptr(X), M, _ptr(Y), _stream(stream), flags),
               "svdq_linear_forward_static")

    def quantize_act(self, X, M: int, codes, scales, xl, stream=None, mode: int = 0):
        self._need_act(M, X=X, codes=codes, scales=scales, xl=xl)
        _check(load().svdq_quantize_act(self._h, _ptr(X), M, _ptr(codes), _ptr(scales), _ptr(xl),
                                        _stream(stream), mode), "svdq_quantize_act")

    def gemm(self, codes, scales, xl, M: int, Y, stream=None, flags: int = 0):
        self._need_act(M, Y=Y, codes=codes, scales=scales, xl=xl)
        _check(load().svdq_gemm(self._h, _ptr(codes), _ptr(scales), _ptr(xl), M, _ptr(Y), _stream(stream),
                                flags), "svdq_gemm")

    def act_scales_to_logical(self, device_layout: np.ndarray, M: int) -> np.ndarray:
        """NVFP4: uint8 [M][K/16] E4M3 bytes; INT4: uint16 [M][K/64] BF16 bits;
        W8A8: float32 [M] (one scale per token)."""
        info = self.info
        if info["format"] == INT4:
            out = np.empty((M, info["K"] // 64), dtype=np.uint16)
        elif info["format"] == W8A8_INT8:
            out = np.empty((M,), dtype=np.float32)
        else:
            out = np.empty((M, info["K"] // 16), dtype=np.uint8)
        src = np.ascontiguousarray(device_layout, dtype=np.uint8)
        _need(src, self.act_scale_bytes(M), "device_layout", device=False)
        _check(load().svdq_act_scales_to_logical(self._h, _ptr(src), M, _ptr(out)), "svdq_act_scales_to_logical")
        return out

    def check(self, stream=None):
        _check(load().svdq_check(self._h, _stream(stream)), "svdq_check")

    def selftest_wait_timeout(self, budget_us: int, stream=None):
        """Enqueue a kernel whose only wait never completes and gives up after
        budget_us; the next check() raises SvdqError with SVDQ_ETIMEOUT."""
        _check(load().svdq_selftest_wait_timeout(self._h, budget_us, _stream(stream)), "svdq_selftest_wait_timeout")


# ---------------------------------------------------------------- fc1 -> fc2 chain

def mlp_workspace_bytes(fc1: Layer, fc2: Layer, M: int, flags: int = 0) -> int:
    """Workspace of mlp_forward / mlp_fc1 for M tokens (svdq_mlp_workspace_bytes)."""
    return int(load().svdq_mlp_workspace_bytes(fc1._h, fc2._h, M, flags))


def mlp_fc1(fc1: Layer, fc2: Layer, X, M: int, codes2, scales2, xl2, workspace, workspace_bytes: int,
            stream=None, flags: int = 0):
    """fc1 with its output handed to fc2 already quantized (svdq_mlp_fc1)."""
    fc1._need_act(M, X=X)
    if M > 0 and xl2 is not None:
        _need(xl2, M * 32 * 2, "xl2")
    fc2._need_act(M, codes=codes2, scales=scales2)
    _need(workspace, workspace_bytes, "workspace")
    _check(load().svdq_mlp_fc1(fc1._h, fc2._h, _ptr(X), M, _ptr(codes2), _ptr(scales2), _ptr(xl2),
                               _ptr(workspace), workspace_bytes, _stream(stream), flags), "svdq_mlp_fc1")


def mlp_forward(fc1: Layer, fc2: Layer, X, M: int, Y, workspace, workspace_bytes: int, stream=None,
                flags: int = 0):
    """fc1 -> [GELU] -> fc2 (svdq_mlp_forward)."""
    fc1._need_act(M, X=X)
    fc2._need_act(M, Y=Y)
    _need(workspace, workspace_bytes, "workspace")
    _check(load().svdq_mlp_forward(fc1._h, fc2._h, _ptr(X), M, _ptr(Y), _ptr(workspace), workspace_bytes,
                                   _stream(stream), flags), "svdq_mlp_forward")
