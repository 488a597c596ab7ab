"""CPU tests of the Python binding's argument checks.

The C ABI takes plain pointers and sizes, so it cannot see how large a buffer
is.  The binding checks PyTorch tensors and NumPy arrays before each call:
device operands are contiguous CUDA tensors, host operands host memory, and
each holds the bytes the call accesses (the sizes include/svdq.h documents:
X [M][K] and Y [M][N] BF16, the activation codes and scales of
svdq_act_code_bytes / svdq_act_scale_bytes, XL [M][32] BF16 or [M][64] with a
LoRA adapter).  A call that passes the checks reaches the library, which
answers a host-only layer's forward with SVDQ_ESTATE; one that fails them
raises ValueError before any pointer is handed over.
"""
import numpy as np
import pytest

import synthetic as syn

import w4a4_diffusion_transformer_b200 as lib


class FakeCuda:
    """Stands in for a CUDA tensor: placement, size and layout, no memory."""

    def __init__(self, nbytes, contiguous=True, cuda=True):
        self.nbytes, self.contiguous, self.is_cuda = nbytes, contiguous, cuda

    def numel(self):
        return self.nbytes // 2

    def element_size(self):
        return 2

    def is_contiguous(self):
        return self.contiguous

    def data_ptr(self):
        return 0x1000


@pytest.fixture(scope="module", autouse=True)
def built():
    from w4a4_diffusion_transformer_b200 import build
    build.build()
    lib.load()


@pytest.fixture(scope="module")
def layer():
    d = syn.custom_layer(61, M=16, K=256, N=128)
    return lib.Layer.prepare(syn.bf16_bits(d["W"]), None, syn.bf16_bits(d["Xc"]), device=-1)


def _state_error(fn):
    with pytest.raises(lib.SvdqError) as e:
        fn()
    assert e.value.status == lib.ESTATE


def test_prepare_shapes():
    d = syn.custom_layer(62, M=16, K=256, N=128)
    W, Xc, b = syn.bf16_bits(d["W"]), syn.bf16_bits(d["Xc"]), syn.bf16_bits(d["bias"])
    for bad in (Xc[:, :128], Xc.reshape(-1), Xc[:1, :1].reshape(1)):
        with pytest.raises(ValueError):
            lib.Layer.prepare(W, b, bad, device=-1)
    with pytest.raises(ValueError):
        lib.Layer.prepare(W, b[:64], Xc, device=-1)
    with pytest.raises(ValueError):
        lib.Layer.prepare(W.reshape(-1), b, Xc, device=-1)
    L = lib.Layer.prepare(W, b, Xc, device=-1)                  # the right shapes still work
    assert L.info["K"] == 256 and L.info["N"] == 128


def test_forward_operand_sizes(layer):
    M, K, N = 16, 256, 128
    X, Y = FakeCuda(M * K * 2), FakeCuda(M * N * 2)
    _state_error(lambda: layer.forward(X, M, Y, FakeCuda(1 << 20), 1 << 20))
    _state_error(lambda: layer.forward_static(X, M, Y))
    for bad_x in (FakeCuda(M * K * 2 - 2), FakeCuda(M * K * 2, contiguous=False), FakeCuda(M * K * 2, cuda=False),
                  np.zeros((M, K), dtype=np.uint16)):
        with pytest.raises(ValueError):
            layer.forward(bad_x, M, Y, FakeCuda(1 << 20), 1 << 20)
    with pytest.raises(ValueError):
        layer.forward(X, M, FakeCuda(M * N * 2 - 2), FakeCuda(1 << 20), 1 << 20)
    with pytest.raises(ValueError):
        layer.forward(X, M, Y, FakeCuda(1 << 10), 1 << 20)        # workspace smaller than its stated size
    with pytest.raises(ValueError):
        layer.forward_static(X, M + 1, Y)
    # raw addresses are the caller's responsibility and pass through
    _state_error(lambda: layer.forward(16, M, 16, 16, 1 << 20))


def test_split_kernels_operand_sizes(layer):
    M, K, N = 33, 256, 128
    X, Y = FakeCuda(M * K * 2), FakeCuda(M * N * 2)
    codes, scales = FakeCuda(layer.act_code_bytes(M)), FakeCuda(layer.act_scale_bytes(M))
    xl = FakeCuda(M * 32 * 2)
    _state_error(lambda: layer.quantize_act(X, M, codes, scales, xl))
    _state_error(lambda: layer.gemm(codes, scales, xl, M, Y))
    with pytest.raises(ValueError):
        layer.quantize_act(X, M, FakeCuda(layer.act_code_bytes(M) - 2), scales, xl)
    with pytest.raises(ValueError):
        layer.gemm(codes, FakeCuda(layer.act_scale_bytes(M) - 2), xl, M, Y)
    with pytest.raises(ValueError):
        layer.gemm(codes, scales, FakeCuda(M * 16 * 2), M, Y)   # XL is [M][32] whatever the rank


def test_xl_width_follows_the_adapter():
    d = syn.custom_layer(63, M=16, K=256, N=128)
    L = lib.Layer.prepare(syn.bf16_bits(d["W"]), None, syn.bf16_bits(d["Xc"]), device=-1)
    M = 8
    X, codes, scales = FakeCuda(M * 256 * 2), FakeCuda(L.act_code_bytes(M)), FakeCuda(L.act_scale_bytes(M))
    rng = np.random.default_rng(3)
    A = syn.bf16_bits(syn.to_bf16(rng.standard_normal((256, 4))))
    B = syn.bf16_bits(syn.to_bf16(rng.standard_normal((4, 128))))
    L.set_lora(A, B, 0.5)
    with pytest.raises(ValueError):
        L.quantize_act(X, M, codes, scales, FakeCuda(M * 32 * 2))
    _state_error(lambda: L.quantize_act(X, M, codes, scales, FakeCuda(M * 64 * 2)))
    L.set_lora(None, None)
    _state_error(lambda: L.quantize_act(X, M, codes, scales, FakeCuda(M * 32 * 2)))
    with pytest.raises(ValueError):
        L.set_lora(A[:128], B, 0.5)                              # A must have K rows
    with pytest.raises(ValueError):
        L.set_lora(A, B[:, :64], 0.5)                            # B must have N columns


def test_host_conversions_check_the_source(layer):
    M = 40
    with pytest.raises(ValueError):
        layer.act_codes_to_logical(np.zeros(layer.act_code_bytes(M) - 1, dtype=np.uint8), M)
    with pytest.raises(ValueError):
        layer.act_scales_to_logical(np.zeros(layer.act_scale_bytes(M) - 1, dtype=np.uint8), M)
    out = layer.act_codes_to_logical(np.zeros(layer.act_code_bytes(M), dtype=np.uint8), M)
    assert out.shape == (M, 128) and not out.any()


def test_mlp_operand_sizes():
    d1 = syn.custom_layer(64, M=8, K=256, N=512)
    d2 = syn.custom_layer(65, M=8, K=512, N=256)
    L1 = lib.Layer.prepare(syn.bf16_bits(d1["W"]), None, syn.bf16_bits(d1["Xc"]), device=-1)
    L2 = lib.Layer.prepare(syn.bf16_bits(d2["W"]), None, syn.bf16_bits(d2["Xc"]), device=-1)
    M = 8
    X, Y, ws = FakeCuda(M * 256 * 2), FakeCuda(M * 256 * 2), FakeCuda(1 << 20)
    _state_error(lambda: lib.mlp_forward(L1, L2, X, M, Y, ws, 1 << 20))
    with pytest.raises(ValueError):
        lib.mlp_forward(L1, L2, FakeCuda(M * 256 * 2 - 2), M, Y, ws, 1 << 20)
    with pytest.raises(ValueError):
        lib.mlp_forward(L1, L2, X, M, FakeCuda(M * 256 * 2 - 2), ws, 1 << 20)
    codes2, scales2 = FakeCuda(L2.act_code_bytes(M)), FakeCuda(L2.act_scale_bytes(M))
    _state_error(lambda: lib.mlp_fc1(L1, L2, X, M, codes2, scales2, FakeCuda(M * 64), ws, 1 << 20))
    with pytest.raises(ValueError):
        lib.mlp_fc1(L1, L2, X, M, codes2, scales2, FakeCuda(M * 64 - 2), ws, 1 << 20)
    with pytest.raises(ValueError):
        lib.mlp_fc1(L1, L2, X, M, FakeCuda(L2.act_code_bytes(M) - 2), scales2, FakeCuda(M * 64), ws, 1 << 20)


def test_layer_as_a_context_manager():
    d = syn.custom_layer(66, M=8, K=128, N=64)
    with lib.Layer.prepare(syn.bf16_bits(d["W"]), None, syn.bf16_bits(d["Xc"]), device=-1) as L:
        assert L.info["K"] == 128
        blob = L.serialize()
    assert L._h is None                                          # freed on leaving the block
    with lib.Layer.deserialize(blob, device=-1) as R:
        assert R.info["N"] == 64
    assert R._h is None
