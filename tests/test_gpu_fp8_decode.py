"""FP8 (E4M3) codes read as codes at decode: ttq_dequant_gemm with 8-bit
codes at T <= 16 against the oracle's FP8 dequantisation, and the FP8
forward at T <= 16, whose workspace holds no binary16 W_hat (blog.lo0.es,
the comparison with FP8 end to end: TTQ derives the scale, the code format
is FP8)."""
import numpy as np
import pytest
import torch

import parity as P
import ttq_oracle
from test_weight_quantization_ttq_b200 import synth, ttq

pytestmark = pytest.mark.gpu

FP8 = ttq.TTQ_QSCHEME_FP8_E4M3


@pytest.fixture(scope="module")
def O():
    return ttq_oracle.get()


CASES = [
    # d, d', T, group, r
    (512, 300, 1, 64, 0),      # PS off (group < 128)
    (1024, 257, 5, 128, 0),    # PS on (T <= 8, group >= 128)
    (768, 130, 16, 256, 8),    # two token tiles, low-rank term
    (4096, 14336, 1, 128, 0),  # the decode workload's shape (sampled rows)
    (576, 64, 9, 32, 0),       # K not a multiple of the 512-channel stage
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "d{}_dp{}_T{}_g{}_r{}".format(*c))
def test_fp8_codes_through_the_decode_product(O, case):
    d, dp, T, group, r = case
    spec = synth.LinearSpec("fp8_dec", d=d, dp=dp, T=T, bits=4, group=group, r=r,
                            n_outliers=5, outlier_lo=20.0, outlier_hi=80.0)
    data = P.inputs(spec)
    X64 = data["X"].astype(np.float64)
    D, Dr, st1 = O.act_norm(X64, *P.params(spec))
    rows = synth.sample_rows(dp, 64)
    W = P.to_dev(data["W"], "bf16")
    Dd = torch.from_numpy(D.astype(np.float32)).cuda()
    codes, sc, ze = ttq.ttq_quantize_weight_ex(W, Dd, 8, group, FP8)
    codes_o, sc_o, ze_o, st2 = O.quantize_fp8(data["W"], D.astype(np.float32), group)
    torch.cuda.synchronize()
    assert np.array_equal(P.u32(codes), codes_o)
    Y_ref = O.project(O.dequant_rows_fp8(codes_o, sc_o, Dr, d, group, rows), X64)
    if r > 0:
        Y_ref = O.lowrank_add(data["A"], data["B"][rows], X64, Y_ref)
    X = P.to_dev(data["X"], "bf16")
    A = P.to_dev(data["A"], "bf16") if r else None
    B = P.to_dev(data["B"], "bf16") if r else None
    Drd = torch.from_numpy(Dr.astype(np.float32)).cuda()
    Y = ttq.ttq_dequant_gemm(codes, sc, ze, Drd, X, A, B, 8, group, y_dtype=torch.float32)
    # the whole forward, whose workspace now has no W_hat at these sizes
    lay = ttq.ttq_workspace_get_layout(d, dp, T, r, 8, group)
    assert lay.wq == 0
    Yf = ttq.ttq_linear_forward(X, W, A, B, spec.p, spec.lam, spec.alpha, 8, group, y_dtype=torch.float32,
                                scheme=FP8)
    torch.cuda.synchronize()
    assert P.y_error(Y.cpu().numpy()[:, rows], Y_ref) <= P.Y_TOL
    assert P.y_error(Yf.cpu().numpy()[:, rows], Y_ref) <= P.Y_TOL


def test_fp8_decode_refuses_long_inputs():
    X = torch.zeros((17, 256), dtype=torch.bfloat16, device="cuda")
    codes = torch.zeros((64, 64), dtype=torch.int32, device="cuda")
    sc = torch.zeros((64, 4), dtype=torch.int16, device="cuda")
    with pytest.raises(ttq.TTQError) as e:
        ttq.ttq_dequant_gemm(codes, sc, sc, None, X, None, None, 8, 64)
    assert e.value.status == ttq.TTQ_ERR_UNSUPPORTED
