"""The Python binding's argument checks (CPU, no device work).

The C ABI receives bare pointers and sizes; the binding derives those sizes
from the tensors it is given, so a tensor whose shape or dtype disagrees
with the others must be refused before any pointer reaches a kernel.  Every
check here fires on CPU tensors, ahead of the device check that would
otherwise reject them.
"""
import pytest
import torch

from test_weight_quantization_ttq_b200 import ttq

bf16, f32, f16 = torch.bfloat16, torch.float32, torch.float16


def t(*shape, dtype=bf16):
    return torch.zeros(shape, dtype=dtype)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    return ttq.lib()


def test_forward_shapes_and_dtypes():
    X, W = t(4, 128), t(64, 128)
    with pytest.raises(ValueError, match="W has shape"):
        ttq.ttq_linear_forward(X, t(64, 256), None, None, 2.0, 1e-3, 0.5, 4, 64)
    with pytest.raises(TypeError, match="W has dtype"):
        ttq.ttq_linear_forward(X, t(64, 128, dtype=f32), None, None, 2.0, 1e-3, 0.5, 4, 64)
    with pytest.raises(ValueError, match="given together"):
        ttq.ttq_linear_forward(X, W, t(8, 128), None, 2.0, 1e-3, 0.5, 4, 64)
    with pytest.raises(ValueError, match="A has shape"):
        ttq.ttq_linear_forward(X, W, t(8, 96), t(64, 8), 2.0, 1e-3, 0.5, 4, 64)
    with pytest.raises(ValueError, match="B has shape"):
        ttq.ttq_linear_forward(X, W, t(8, 128), t(64, 16), 2.0, 1e-3, 0.5, 4, 64)
    with pytest.raises(TypeError, match="A has dtype"):
        ttq.ttq_linear_forward(X, W, t(8, 128, dtype=f32), t(64, 8), 2.0, 1e-3, 0.5, 4, 64)
    with pytest.raises(ValueError, match="Y has shape"):
        ttq.ttq_linear_forward(X, W, None, None, 2.0, 1e-3, 0.5, 4, 64, Y=t(4, 32))
    with pytest.raises(TypeError, match="X has dtype"):
        ttq.ttq_linear_forward(t(4, 128, dtype=f16), t(64, 128, dtype=f16), None, None, 2.0, 1e-3,
                               0.5, 4, 64)
    with pytest.raises(ValueError, match="X must be 2-D"):
        ttq.ttq_linear_forward(t(128), W, None, None, 2.0, 1e-3, 0.5, 4, 64)
    # consistent shapes get as far as the device check
    with pytest.raises(ValueError, match="CUDA tensor"):
        ttq.ttq_linear_forward(X, W, t(8, 128), t(64, 8), 2.0, 1e-3, 0.5, 4, 64)


def test_quantizer_outputs():
    W = t(64, 256)
    with pytest.raises(ValueError, match="D must hold 256"):
        ttq.ttq_quantize_weight(W, t(128, dtype=f32), 4, 64)
    with pytest.raises(ValueError, match="D must hold 256"):
        ttq.ttq_quantize_weight(W, t(256, dtype=bf16), 4, 64)
    # 4-bit codes of a 64 x 256 weight span 64 * 32 words
    with pytest.raises(ValueError, match="codes spans"):
        ttq.ttq_quantize_weight(W, None, 4, 64, codes=t(64, 31, dtype=torch.int32))
    with pytest.raises(ValueError, match="scales spans"):
        ttq.ttq_quantize_weight(W, None, 4, 64, scales=t(64, 3, dtype=torch.int16))
    with pytest.raises(ValueError, match="zeros spans"):
        ttq.ttq_quantize_weight_ex(W, None, 2, 32, ttq.TTQ_QSCHEME_SYMMETRIC,
                                   zeros=t(63, 8, dtype=torch.int16))
    with pytest.raises(ValueError, match="W_hat has shape"):
        ttq.ttq_quantize_dequant_weight(W, None, 4, 64, W_hat=t(64, 255, dtype=f16))
    with pytest.raises(TypeError, match="W_hat has dtype"):
        ttq.ttq_quantize_weight_ex(W, None, 8, 64, ttq.TTQ_QSCHEME_FP8_E4M3, W_hat=t(64, 256))
    with pytest.raises(ttq.TTQError):
        ttq.ttq_quantize_weight(W, None, 4, 0)
    # a code buffer of another 4-byte type and the exact size passes the check
    with pytest.raises(ValueError, match="CUDA tensor"):
        ttq.ttq_quantize_weight(W, None, 3, 64, codes=t(64 * 24, dtype=f32))


def test_statistic_and_scaling():
    X = t(5, 64)
    with pytest.raises(ValueError, match="D_rsqrt must hold 64"):
        ttq.ttq_act_norm(X, 2.0, 1e-3, 0.5, D_rsqrt=t(63, dtype=f32))
    with pytest.raises(ValueError, match="Xs has shape"):
        ttq.ttq_act_norm_scale(X, 2.0, 1e-3, 0.5, Xs=t(5, 32, dtype=f16))
    with pytest.raises(TypeError, match="Xs has dtype"):
        ttq.ttq_scale_activations(X, None, Xs=t(5, 64))
    with pytest.raises(ValueError, match="D must hold 64"):
        ttq.ttq_act_norm_noalloc(X, 2.0, 1e-3, 0.5, D=t(64, dtype=torch.float64))


def test_products():
    with pytest.raises(ValueError, match="Xs has shape"):
        ttq.ttq_dequantized_gemm(t(32, 64, dtype=f16), t(8, 128, dtype=f16))
    with pytest.raises(ValueError, match="Y has shape"):
        ttq.ttq_dequantized_gemm(t(32, 64, dtype=f16), t(8, 64, dtype=f16), Y=t(32, 8))
    codes, sc = t(32, 8, dtype=torch.int32), t(32, 1, dtype=torch.int16)
    X = t(8, 64, dtype=f16)
    with pytest.raises(ValueError, match="codes spans"):
        ttq.ttq_dequant_gemm(t(32, 7, dtype=torch.int32), sc, sc, None, X, None, None, 4, 64)
    with pytest.raises(ValueError, match="scales spans"):
        ttq.ttq_dequant_gemm(codes, t(31, 1, dtype=torch.int16), sc, None, X, None, None, 4, 64)
    with pytest.raises(ValueError, match="D_rsqrt must hold 64"):
        ttq.ttq_dequant_gemm(codes, sc, sc, t(32, dtype=f32), X, None, None, 4, 64)
    Xb = t(8, 64)
    with pytest.raises(ValueError, match="B has shape"):
        ttq.ttq_dequant_gemm(codes, sc, sc, None, Xb, t(8, 64), t(8, 8), 4, 64)


def test_lowrank_init():
    W = t(100, 64)
    with pytest.raises(ValueError, match="Omega has shape"):
        ttq.ttq_lowrank_init(W, 8, t(100, 16, dtype=f32))
    with pytest.raises(TypeError, match="Omega has dtype"):
        ttq.ttq_lowrank_init(W, 8, t(64, 16))
    with pytest.raises(ValueError, match="B has shape"):
        ttq.ttq_lowrank_init(W, 8, t(64, 16, dtype=f32), B=t(100, 16))
    with pytest.raises(TypeError, match="W_res has dtype"):
        ttq.ttq_lowrank_init(W, 8, t(64, 16, dtype=f32), W_res=t(100, 64, dtype=f32))
