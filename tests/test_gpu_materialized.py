"""For more than 256 tokens the forward writes the dequantised weight
s (q - z) in binary16 once (in place of the codes) and runs the product on
it as a plain tensor-core operand.  Those operand values must be exactly
the dequantisation of the codes, scales and zeros that the quantiser gives
for the call's D (TTQ paper, section 2.1: W_hat = Q[W D^(1/2)] D^(-1/2),
with the D^(-1/2) factor carried by X), and the product must equal the one
that dequantises inside the GEMM (ttq_dequant_gemm) on the same operands."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import parity as P
import ttq_oracle
from test_weight_quantization_ttq_b200 import synth, ttq

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def O():
    return ttq_oracle.get()


def _spec(name, d, dp, T, bits, group, dtype="bf16", r=0):
    return synth.LinearSpec(name, d=d, dp=dp, T=T, bits=bits, group=group, dtype=dtype, r=r,
                            n_outliers=3, outlier_lo=20.0, outlier_hi=80.0)


CASES = [
    _spec("int4_g128", d=1024, dp=640, T=300, bits=4, group=128),
    _spec("int3_g32_ragged", d=96 * 8, dp=200, T=333, bits=3, group=32),
    _spec("int2_g64_lowrank", d=512, dp=264, T=520, bits=2, group=64, r=24),
    _spec("int4_f32_lowrank", d=448, dp=96, T=257, bits=4, group=64, dtype="f32", r=16),
]


@pytest.mark.parametrize("spec", CASES, ids=lambda s: s.name)
def test_materialized_weight_is_the_dequantised_codes(O, spec):
    data = P.inputs(spec)
    dt = ttq.TTQ_F32 if spec.dtype == "f32" else ttq.TTQ_BF16
    X = P.to_dev(data["X"], spec.dtype)
    W = P.to_dev(data["W"], spec.dtype)
    A = P.to_dev(data["A"], spec.dtype) if spec.r else None
    B = P.to_dev(data["B"], spec.dtype) if spec.r else None
    ws = ttq.new_workspace(spec.d, spec.dp, spec.T, spec.r, spec.bits, spec.group, dt)
    Y = ttq.ttq_linear_forward(X, W, A, B, spec.p, spec.lam, spec.alpha, spec.bits, spec.group,
                               ws=ws, y_dtype=torch.float32)
    torch.cuda.synchronize()
    st, flags = ttq.ttq_get_status(ws)
    assert st == ttq.TTQ_OK, flags
    v = ttq.workspace_views(ws, spec.d, spec.dp, spec.T, spec.r, spec.bits, spec.group, dt)
    assert "wq" in v
    # the forward keeps W_hat and no codes; the quantiser, given the
    # forward's D, gives the codes W_hat must be the dequantisation of
    codes, scales, zeros = ttq.ttq_quantize_weight(W, v["D"], spec.bits, spec.group)
    torch.cuda.synchronize()
    q = O.unpack(P.u32(codes), spec.d, spec.bits).astype(np.float64)
    s = P.u16(scales).view(np.float16).astype(np.float64)
    z = P.u16(zeros).view(np.float16).astype(np.float64)
    k = np.arange(spec.d) // spec.group
    # s (q - z) is exact in float64; one rounding to binary16
    ref = (s[:, k] * (q - z[:, k])).astype(np.float16)
    assert np.array_equal(v["wq"].cpu().numpy().view(np.uint16), ref.view(np.uint16))
    # the same product from the codes, dequantised inside the GEMM
    if spec.r == 0:
        Y2 = ttq.ttq_dequant_gemm(codes, scales, zeros, None, v["xh"], None, None,
                                  spec.bits, spec.group, y_dtype=torch.float32)
        torch.cuda.synchronize()
        rms = float(Y2.double().pow(2).mean().sqrt())
        assert float((Y - Y2).abs().max()) <= 1e-5 * rms
    rows = synth.sample_rows(spec.dp, 48)
    ref_y = O.forward(data["X"].astype(np.float64), data["W"], *P.params(spec), spec.bits, spec.group,
                      A=data.get("A"), B=data.get("B"), rows=rows)["Y"]
    assert P.y_error(Y.cpu().numpy()[:, rows], ref_y) <= P.Y_TOL



@pytest.mark.parametrize("spec", [synth.C2.with_(T=300, dp=640),
                                  # few output tiles: the product splits along K
                                  synth.C2.with_(T=333, dp=200)], ids=lambda s: f"dp{s.dp}-T{s.T}")
def test_composed_materialized_steps_equal_forward(spec):
    """ttq_act_norm_scale -> ttq_quantize_dequant_weight -> ttq_dequantized_gemm
    is the forward for more than 256 tokens, bit for bit (also where the
    product is split along K and its partial sums are added in split order)."""
    data = P.inputs(spec)
    X, W = P.to_dev(data["X"], "bf16"), P.to_dev(data["W"], "bf16")
    Y = ttq.ttq_linear_forward(X, W, None, None, spec.p, spec.lam, spec.alpha, spec.bits, spec.group,
                               y_dtype=torch.float32)
    D, Dr, Xs = ttq.ttq_act_norm_scale(X, spec.p, spec.lam, spec.alpha)
    codes, sc, ze, W_hat = ttq.ttq_quantize_dequant_weight(W, D, spec.bits, spec.group)
    Y2 = ttq.ttq_dequantized_gemm(W_hat, Xs, y_dtype=torch.float32)
    Yb = ttq.ttq_dequantized_gemm(W_hat, Xs, y_dtype=torch.bfloat16)
    codes1, sc1, ze1 = ttq.ttq_quantize_weight(W, D, spec.bits, spec.group)
    # W_hat alone (no codes, scales or zeros), as the forward writes it
    _, _, _, W_hat1 = ttq.ttq_quantize_dequant_weight(W, D, spec.bits, spec.group, with_codes=False)
    torch.cuda.synchronize()
    assert torch.equal(Y, Y2)
    assert torch.equal(Yb, Y2.to(torch.bfloat16))
    assert torch.equal(codes, codes1) and torch.equal(sc, sc1) and torch.equal(ze, ze1)
    assert torch.equal(W_hat1.view(torch.int16), W_hat.view(torch.int16))
