"""The single-pass decode product (ttq_quantize_gemm) against the oracle.

For a few tokens the layer's test-time steps outweigh the product
(gist.science/zh/paper/2603.19296, section 2.3), so one kernel reads bf16 W
once, quantises it in the quantiser's binary32 order and multiplies in the
same pass.  Its codes, scales and zeros (stored on request) must be the
oracle's bit for bit on a shared D; Y must be within the layer's tolerance
of the oracle's; the forward at a few tokens must be this kernel's result.
"""
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


def _spec(name, d, dp, T, bits, group, r=0, seed=0, n_out=3):
    return synth.LinearSpec(name, d=d, dp=dp, T=T, bits=bits, group=group, r=r, n_outliers=n_out,
                            outlier_lo=20.0, outlier_hi=80.0, seed=seed)


# shapes: ragged row tiles (d' not a multiple of 128), tiles shared by two
# or more CTAs (few units per CTA), every bit width and group size, 1 to 16
# tokens (one and two token tiles), the low-rank term, and the full decode
# workloads (d' = 14336 INT4 g128; the 70B-like d' = 28672 INT2 g64 r = 64)
CASES = [
    _spec("t1_int4_g128", 256, 200, 1, 4, 128),
    _spec("t9_int2_g64_lr8", 384, 130, 9, 2, 64, r=8),
    _spec("t3_int3_g32", 256, 129, 3, 3, 32),
    _spec("t16_int4_g64_lr16", 128, 257, 16, 4, 64, r=16),
    _spec("t2_int3_g128", 512, 64, 2, 3, 128),
    _spec("t5_int4_g32_lr24", 1024, 1000, 5, 4, 32, r=24),
    _spec("t8_int2_g128", 2048, 777, 8, 2, 128, seed=3),
    _spec("t13_int3_g64", 640, 385, 13, 3, 64, seed=4),
    synth.C4.with_(T=1),
    synth.C4.with_(T=16),
    synth.C5.with_(T=1),
    synth.C5.with_(T=16),
]


@pytest.mark.parametrize("spec", CASES, ids=lambda s: f"{s.name}-T{s.T}")
def test_single_pass_matches_oracle(O, spec):
    data = P.inputs_shared_w(spec)
    X64 = data["X"].astype(np.float64)
    pf, lf, af = P.params(spec)
    D_ref, Dr_ref, st = O.act_norm(X64, pf, lf, af)
    assert st == 0
    D32 = D_ref.astype(np.float32)          # both sides quantise with this D
    codes_ref, sc_ref, ze_ref, st = O.quantize(data["W"], D32, spec.bits, spec.group)
    assert st == 0
    X = P.to_dev(data["X"], "bf16")
    W = P.to_dev(data["W"], "bf16")
    A = P.to_dev(data["A"], "bf16") if spec.r else None
    B = P.to_dev(data["B"], "bf16") if spec.r else None
    Dd = torch.from_numpy(D32).cuda()
    Drd = torch.from_numpy(Dr_ref.astype(np.float32)).cuda()
    Xs = ttq.ttq_scale_activations(X, Drd)
    cb, sb = spec.d * spec.bits // 32, spec.d // spec.group
    codes = torch.empty((spec.dp, cb), dtype=torch.int32, device="cuda")
    sc = torch.empty((spec.dp, sb), dtype=torch.int16, device="cuda")
    ze = torch.empty((spec.dp, sb), dtype=torch.int16, device="cuda")
    ws = ttq.new_workspace(spec.d, spec.dp, spec.T, spec.r, spec.bits, spec.group)
    Y = ttq.ttq_quantize_gemm(W, Dd, Xs, A, B, X, spec.bits, spec.group, ws=ws, y_dtype=torch.float32,
                              codes=codes, scales=sc, zeros=ze)
    # without the codes: the same arithmetic, the same Y; and a bf16 Y is the
    # fp32 one rounded once
    Y2 = ttq.ttq_quantize_gemm(W, Dd, Xs, A, B, X, spec.bits, spec.group, ws=ws, y_dtype=torch.float32)
    Yb = ttq.ttq_quantize_gemm(W, Dd, Xs, A, B, X, spec.bits, spec.group, ws=ws, y_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    st, flags = ttq.ttq_get_status(ws)
    assert st == ttq.TTQ_OK, flags
    assert np.array_equal(P.u32(codes), codes_ref)
    assert np.array_equal(P.u16(sc), sc_ref)
    assert np.array_equal(P.u16(ze), ze_ref)
    assert torch.equal(Y, Y2)
    assert torch.equal(Yb, Y.to(torch.bfloat16))
    # every tile ticket is back at zero after the calls
    L = ttq.ttq_workspace_get_layout(spec.d, spec.dp, spec.T, spec.r, spec.bits, spec.group)
    assert L.tickets and not ws[L.tickets: L.tickets + 4 * ((spec.dp + 127) // 128)].any()
    rows = synth.sample_rows(spec.dp, 96)
    What = O.dequant_rows(codes_ref, sc_ref, ze_ref, Dr_ref, spec.d, spec.bits, spec.group, rows)
    Y_ref = O.project(What, X64)
    if spec.r:
        Y_ref = O.lowrank_add(data["A"], data["B"][rows], X64, Y_ref)
    err = P.y_error(Y.cpu().numpy()[:, rows], Y_ref)
    assert err <= P.Y_TOL, err


def test_single_pass_is_the_forward_and_deterministic():
    """The forward at a few tokens is ttq_act_norm_scale followed by this
    kernel, bit for bit, and two calls give the same bits."""
    spec = _spec("fwd", 1024, 900, 4, 4, 128, r=16, n_out=10)
    data = P.inputs(spec)
    X, W = P.to_dev(data["X"], "bf16"), P.to_dev(data["W"], "bf16")
    A, B = P.to_dev(data["A"], "bf16"), P.to_dev(data["B"], "bf16")
    Y = ttq.ttq_linear_forward(X, W, A, B, spec.p, spec.lam, spec.alpha, spec.bits, spec.group,
                               y_dtype=torch.float32)
    D, Dr, Xs = ttq.ttq_act_norm_scale(X, spec.p, spec.lam, spec.alpha)
    Y1 = ttq.ttq_quantize_gemm(W, D, Xs, A, B, X, spec.bits, spec.group, y_dtype=torch.float32)
    Y2 = ttq.ttq_quantize_gemm(W, D, Xs, A, B, X, spec.bits, spec.group, y_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(Y, Y1) and torch.equal(Y1, Y2)


def test_single_pass_rejects_what_it_does_not_cover():
    W = torch.zeros((64, 256), dtype=torch.bfloat16, device="cuda")
    D = torch.ones(256, device="cuda")
    for T, group, d in ((17, 128, 256), (4, 256, 256), (4, 64, 192)):
        Ww = torch.zeros((64, d), dtype=torch.bfloat16, device="cuda")
        Xs = torch.zeros((T, d), dtype=torch.float16, device="cuda")
        with pytest.raises(ttq.TTQError) as e:
            ttq.ttq_quantize_gemm(Ww, torch.ones(d, device="cuda"), Xs, None, None, None, 4, group)
        assert e.value.status == ttq.TTQ_ERR_UNSUPPORTED, (T, group, d)
    del W, D
