"""FP8 (E4M3) codes on the GPU (TTQ_QSCHEME_FP8_E4M3) against the oracle.

The quantiser's codes, scales and zeros must match the oracle bit for bit
(both take the E4M3 rounding of the same binary32 product), and its binary16
s * e4m3(q) must equal that product rounded once.  The forward, which always
materialises the binary16 weight for this scheme, must meet the layer's
tolerance against the oracle's forward on FP8 codes.
"""
import numpy as np
import pytest
import torch

import parity as P
import ttq_oracle
from test_weight_quantization_ttq_b200 import synth
from test_weight_quantization_ttq_b200 import ttq

pytestmark = pytest.mark.gpu

FP8 = ttq.TTQ_QSCHEME_FP8_E4M3


@pytest.fixture(scope="module")
def O():
    return ttq_oracle.get()


def _e4m3_to_f16(codes_bytes: np.ndarray) -> np.ndarray:
    """E4M3 values (from the format's definition) as float16; exact."""
    c = codes_bytes.astype(np.int64)
    e, m = (c >> 3) & 15, c & 7
    v = np.where(e == 0, m / 8 * 2.0 ** -6, (1 + m / 8) * np.exp2(e - 7.0))
    v = np.where(c & 0x80, -v, v)
    return v.astype(np.float16)


QUANT_CASES = [
    # d', d, group, dtype
    (37, 512, 32, "bf16"),
    (64, 256, 64, "bf16"),
    (130, 1024, 128, "bf16"),
    (16, 768, 256, "bf16"),
    (9, 96, 32, "f32"),
]


@pytest.mark.parametrize("case", QUANT_CASES, ids=lambda c: "dp{}_d{}_g{}_{}".format(*c))
def test_fp8_quantizer_bit_exact(O, case):
    dp, d, group, dtype = case
    spec = synth.LinearSpec("fp8_q", d=d, dp=dp, T=4, bits=4, group=group, dtype=dtype,
                            n_outliers=3, outlier_lo=20.0, outlier_hi=80.0)
    data = P.inputs(spec)
    g = np.random.Generator(np.random.PCG64(dp * 7 + d))
    D32 = np.exp(g.uniform(-4.0, 4.0, d)).astype(np.float32)
    codes_o, sc_o, ze_o, st = O.quantize_fp8(data["W"], D32, group)
    assert st == 0
    W = P.to_dev(data["W"], dtype)
    Dd = torch.from_numpy(D32).cuda()
    W_hat = torch.empty((dp, d), dtype=torch.float16, device="cuda")
    codes, sc, ze = ttq.ttq_quantize_weight_ex(W, Dd, 8, group, FP8, W_hat=W_hat)
    torch.cuda.synchronize()
    assert np.array_equal(P.u32(codes), codes_o)
    assert np.array_equal(P.u16(sc), sc_o)
    assert np.array_equal(P.u16(ze), ze_o) and not ze_o.any()
    # W_hat = binary16(s * e4m3(q)): both factors are binary16, so float32
    # holds their product exactly and one rounding to binary16 follows
    q = codes_o.view(np.uint8).reshape(dp, d)
    s16 = np.repeat(sc_o.view(np.float16), group, axis=1)
    want = (s16.astype(np.float32) * _e4m3_to_f16(q).astype(np.float32)).astype(np.float16)
    assert np.array_equal(W_hat.cpu().numpy().view(np.uint16), want.view(np.uint16))
    # W_hat alone (no codes, scales or zeros), as the forward writes it above 16 tokens
    W_hat1 = torch.empty_like(W_hat)
    ttq.ttq_quantize_weight_ex(W, Dd, 8, group, FP8, W_hat=W_hat1, with_codes=False)
    torch.cuda.synchronize()
    assert torch.equal(W_hat1.view(torch.int16), W_hat.view(torch.int16))


FORWARD_CASES = [
    # d, d', T, group, r
    (512, 300, 1, 64, 0),
    (1024, 257, 16, 128, 16),
    (768, 512, 300, 32, 0),
]


@pytest.mark.parametrize("case", FORWARD_CASES, ids=lambda c: "d{}_dp{}_T{}_g{}_r{}".format(*c))
def test_fp8_forward_matches_oracle(O, case):
    d, dp, T, group, r = case
    spec = synth.LinearSpec("fp8_fwd", d=d, dp=dp, T=T, bits=4, group=group, r=r,
                            n_outliers=5, outlier_lo=20.0, outlier_hi=80.0)
    data = P.inputs(spec)
    X64 = data["X"].astype(np.float64)
    D, Dr, st1 = O.act_norm(X64, *P.params(spec))
    codes, sc, ze, st2 = O.quantize_fp8(data["W"], D.astype(np.float32), group)
    assert st1 == 0 and st2 == 0
    rows = synth.sample_rows(dp, 64)
    Y_ref = O.project(O.dequant_rows_fp8(codes, sc, Dr, d, group, rows), X64)
    if r > 0:
        Y_ref = O.lowrank_add(data["A"], data["B"][rows], X64, Y_ref)
    X = P.to_dev(data["X"], "bf16")
    W = P.to_dev(data["W"], "bf16")
    A = P.to_dev(data["A"], "bf16") if r else None
    B = P.to_dev(data["B"], "bf16") if r else None
    ws = ttq.new_workspace(d, dp, T, r, 8, group)
    Y = ttq.ttq_linear_forward(X, W, A, B, spec.p, spec.lam, spec.alpha, 8, group, ws=ws,
                               y_dtype=torch.float32, scheme=FP8)
    torch.cuda.synchronize()
    st, flags = ttq.ttq_get_status(ws)
    assert st == ttq.TTQ_OK, flags
    err = P.y_error(Y.cpu().numpy()[:, rows], Y_ref)
    assert err <= P.Y_TOL, err
