"""The symmetric code scheme (blog.lo0.es "Test-time quantization ...",
section "The maths that matter": levels +-(2^(b-1) - 1), scale max|x| over
2^(b-1) - 1) on the GPU against the oracle: codes, scales and zeros bit for
bit on a shared D, the dequantised binary16 weight, and the whole forward
through both products (codes dequantised in the GEMM for T <= 256, the
materialised binary16 weight above)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import parity as P
import ttq_oracle
from test_weight_quantization_ttq_b200 import synth, ttq

pytestmark = pytest.mark.gpu
SYM = ttq.TTQ_QSCHEME_SYMMETRIC


@pytest.fixture(scope="module")
def O():
    return ttq_oracle.get()


def _spec(name, d, dp, T, bits, group, dtype="bf16", r=0, seed=0):
    return synth.LinearSpec(name, d=d, dp=dp, T=T, bits=bits, group=group, dtype=dtype, r=r,
                            n_outliers=3, outlier_lo=20.0, outlier_hi=80.0, seed=seed)


QUANT_CASES = [synth.C1, synth.C2] + [
    _spec(f"b{b}_g{g}", d=512, dp=96, T=32, bits=b, group=g, seed=b * 7 + g)
    for b in (2, 3, 4) for g in (32, 64, 128, 256)
]


@pytest.mark.parametrize("spec", QUANT_CASES, ids=lambda s: s.name)
def test_symmetric_quantize_bit_exact(O, spec):
    data = P.inputs(spec)
    D_ref, _, _ = O.act_norm(data["X"].astype(np.float64), *P.params(spec))
    D32 = D_ref.astype(np.float32)
    codes_ref, sc_ref, ze_ref, st = O.quantize(data["W"], D32, spec.bits, spec.group, symmetric=True)
    assert st == 0
    W = P.to_dev(data["W"], spec.dtype)
    W_hat = torch.empty(W.shape, dtype=torch.float16, device="cuda")
    codes, sc, ze = ttq.ttq_quantize_weight_ex(W, torch.from_numpy(D32).cuda(), spec.bits, spec.group,
                                               SYM, W_hat=W_hat)
    torch.cuda.synchronize()
    assert np.array_equal(P.u32(codes), codes_ref)
    assert np.array_equal(P.u16(sc), sc_ref)
    assert np.array_equal(P.u16(ze), ze_ref)
    q = O.unpack(codes_ref, spec.d, spec.bits).astype(np.float64)
    s = sc_ref.view(np.float16).astype(np.float64)
    z = ze_ref.view(np.float16).astype(np.float64)
    k = np.arange(spec.d) // spec.group
    ref_wh = (s[:, k] * (q - z[:, k])).astype(np.float16)
    assert np.array_equal(W_hat.cpu().numpy().view(np.uint16), ref_wh.view(np.uint16))


def test_symmetric_worked_example(O):
    """The blog's INT4 group of unit magnitudes with one 30: s is the
    binary16 value just above 30/7 and the 30 takes the top level."""
    row = np.ones((1, 32), np.float32)
    row[0, 1::2] = -1.0
    row[0, 5] = 30.0
    W = torch.from_numpy(row).cuda()
    codes, sc, ze = ttq.ttq_quantize_weight_ex(W, None, 4, 32, SYM)
    ref = O.quantize(row, None, 4, 32, symmetric=True)
    torch.cuda.synchronize()
    assert np.array_equal(P.u32(codes), ref[0]) and np.array_equal(P.u16(sc), ref[1])
    s = float(P.u16(sc).view(np.float16)[0, 0])
    assert 30 / 7 <= s <= 30 / 7 * (1 + 2 ** -10)
    assert O.unpack(P.u32(codes), 32, 4)[0, 5] == 15


FORWARD_CASES = [
    _spec("decode_T16", d=1024, dp=640, T=16, bits=4, group=128),
    _spec("prefill_T300", d=1024, dp=640, T=300, bits=4, group=128),
    _spec("int2_lowrank_T64", d=512, dp=264, T=64, bits=2, group=64, r=16),
    _spec("int3_lowrank_T520", d=768, dp=200, T=520, bits=3, group=32, r=24),
]


@pytest.mark.parametrize("spec", FORWARD_CASES, ids=lambda s: s.name)
def test_symmetric_forward_matches_oracle(O, spec):
    data = P.inputs(spec)
    rows = synth.sample_rows(spec.dp, 48)
    ref = O.forward(data["X"].astype(np.float64), data["W"], *P.params(spec), spec.bits, spec.group,
                    A=data.get("A"), B=data.get("B"), rows=rows, symmetric=True)
    assert ref["status"] == 0
    X, W = P.to_dev(data["X"], spec.dtype), P.to_dev(data["W"], spec.dtype)
    A = P.to_dev(data["A"], spec.dtype) if spec.r else None
    B = P.to_dev(data["B"], spec.dtype) if spec.r else None
    ws = ttq.new_workspace(spec.d, spec.dp, spec.T, spec.r, spec.bits, spec.group)
    Y = ttq.ttq_linear_forward(X, W, A, B, spec.p, spec.lam, spec.alpha, spec.bits, spec.group, ws=ws,
                               y_dtype=torch.float32, scheme=SYM)
    torch.cuda.synchronize()
    st, flags = ttq.ttq_get_status(ws)
    assert st == ttq.TTQ_OK, flags
    v = ttq.workspace_views(ws, spec.d, spec.dp, spec.T, spec.r, spec.bits, spec.group)
    codes_d, sc_d, ze_d = v["codes"], v["scales"], v["zeros"]
    if "wq" in v:
        # the forward kept the binary16 W_hat only: the quantiser, given the
        # forward's D, gives the codes, and W_hat must be their dequantisation
        codes_d, sc_d, ze_d = ttq.ttq_quantize_weight_ex(W, v["D"], spec.bits, spec.group, SYM)
        torch.cuda.synchronize()
        q = O.unpack(P.u32(codes_d), spec.d, spec.bits).astype(np.float64)
        k = np.arange(spec.d) // spec.group
        sv = P.u16(sc_d).view(np.float16).astype(np.float64)[:, k]
        zv = P.u16(ze_d).view(np.float16).astype(np.float64)[:, k]
        assert np.array_equal(v["wq"].cpu().numpy().view(np.uint16),
                              (sv * (q - zv)).astype(np.float16).view(np.uint16))
    same_d = v["D"].cpu().numpy() == ref["D"].astype(np.float32)
    group_ok = same_d.reshape(-1, spec.group).all(axis=1)
    assert group_ok.mean() >= 0.99
    wpg = spec.group * spec.bits // 32
    codes = P.u32(codes_d).reshape(spec.dp, -1, wpg)
    assert np.array_equal(codes[:, group_ok], ref["codes"].reshape(spec.dp, -1, wpg)[:, group_ok])
    assert np.array_equal(P.u16(sc_d)[:, group_ok], ref["scales"][:, group_ok])
    assert np.all(P.u16(ze_d).view(np.float16) == 2 ** (spec.bits - 1))
    assert P.y_error(Y.cpu().numpy()[:, rows], ref["Y"]) <= P.Y_TOL
