"""The forward computes the statistic D and the binary16 operand X D^(-1/2)
either in one kernel (when each token split's rows fit in registers: the
splits of a 128-channel column block then form one thread-block cluster and
merge through distributed shared memory) or in two kernels.  Both must give
exactly what the stand-alone entry points ttq_act_norm and
ttq_scale_activations give (TTQ paper, section 2.1: D_ii = (||X_i,:||_p +
lambda)^alpha; section 2.2: the product runs on X D^(-1/2))."""
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


def _spec(name, d, dp, T, p=2.0, alpha=0.5, dtype="bf16", r=0, bits=4, group=32):
    return synth.LinearSpec(name, d=d, dp=dp, T=T, bits=bits, group=group, dtype=dtype, r=r, p=p,
                            lam=1e-3, alpha=alpha, n_outliers=3, outlier_lo=20.0,
                            outlier_hi=80.0)


CASES = [
    synth.C2.with_(dp=256),                                  # fused: 32 clusters of 8 splits of 256 rows
    _spec("ragged_channels_p3", d=96, dp=64, T=19, p=3.0),   # one partial column block, any p
    _spec("ragged_block_p1", d=288, dp=64, T=1000, p=1.0, alpha=0.25),
    _spec("cluster_of_5", d=4096, dp=64, T=150),              # 5 splits of 30 rows
    _spec("f32_lowrank", d=448, dp=96, T=77, dtype="f32", r=16),
    _spec("f32_two_kernel", d=1024, dp=64, T=2048, dtype="f32"),  # 256 rows: too many for f32
    _spec("one_token", d=4096, dp=64, T=1),
    _spec("wide", d=8192, dp=64, T=2048),                     # 64 clusters, more than one wave
    _spec("long_two_kernel", d=4096, dp=64, T=4096, alpha=0.25),
    _spec("no_tokens", d=512, dp=64, T=0),
]


def _dt(spec):
    return ttq.TTQ_F32 if spec.dtype == "f32" else ttq.TTQ_BF16


@pytest.mark.parametrize("spec", CASES, ids=lambda s: f"{s.name}-d{s.d}-T{s.T}")
def test_forward_statistic_equals_standalone(spec):
    """Forward's workspace D, D^(-1/2) and X D^(-1/2), and ttq_act_norm_scale's
    outputs, equal ttq_act_norm followed by ttq_scale_activations bit for bit."""
    data = P.inputs(spec)
    X = P.to_dev(data["X"], spec.dtype)
    W = P.to_dev(data["W"], spec.dtype)
    A = P.to_dev(data["A"], spec.dtype) if spec.r else None
    B = P.to_dev(data["B"], spec.dtype) if spec.r else None
    ws = ttq.new_workspace(spec.d, spec.dp, spec.T, spec.r, spec.bits, spec.group, _dt(spec))
    ttq.ttq_linear_forward(X, W, A, B, spec.p, spec.lam, spec.alpha, spec.bits, spec.group, ws=ws,
                           y_dtype=torch.float32)
    D, Dr = ttq.ttq_act_norm(X, spec.p, spec.lam, spec.alpha)
    Xs = ttq.ttq_scale_activations(X, Dr)
    ws1 = ttq.new_workspace(spec.d, 0, spec.T, 0, 4, 32, _dt(spec))
    D1, Dr1, Xs1 = ttq.ttq_act_norm_scale(X, spec.p, spec.lam, spec.alpha, ws=ws1)
    D2, Dr2, Xs2 = ttq.ttq_act_norm_scale(X, spec.p, spec.lam, spec.alpha, ws=ws1, copy_out=False)
    torch.cuda.synchronize()
    for w in (ws, ws1):
        st, flags = ttq.ttq_get_status(w)
        assert st == ttq.TTQ_OK, flags
    v = ttq.workspace_views(ws, spec.d, spec.dp, spec.T, spec.r, spec.bits, spec.group, _dt(spec))
    for d_, dr_, xs_ in ((v["D"], v["D_rsqrt"], v["xh"]), (D1, Dr1, Xs1), (D2, Dr2, Xs2)):
        assert torch.equal(d_, D)
        assert torch.equal(dr_, Dr)
        assert torch.equal(xs_.view(torch.int16), Xs.view(torch.int16))


def test_forward_lowrank_f32_matches_oracle(O):
    """float32 X with a low-rank pair: the bf16 copy of X that the A X product
    reads is written by the statistic pass."""
    spec = _spec("f32_lowrank", d=448, dp=96, T=77, dtype="f32", r=16)
    data = P.inputs(spec)
    ref = O.forward(data["X"].astype(np.float64), data["W"], *P.params(spec), spec.bits,
                    spec.group, A=data["A"], B=data["B"])
    Y = ttq.ttq_linear_forward(*(P.to_dev(data[k], "f32") for k in ("X", "W", "A", "B")),
                               spec.p, spec.lam, spec.alpha, spec.bits, spec.group,
                               y_dtype=torch.float32)
    torch.cuda.synchronize()
    assert P.y_error(Y.cpu().numpy(), ref["Y"]) <= P.Y_TOL


def test_workspace_reused_across_shapes():
    """The statistic's merge tickets are left at zero, so one workspace
    serves calls of different grid sizes in a row."""
    big = synth.C2.with_(dp=256)
    ws = ttq.new_workspace(big.d, big.dp, big.T, 0, big.bits, big.group, ttq.TTQ_BF16)
    outs = []
    for spec in (big, _spec("small", d=288, dp=64, T=1000), big, _spec("tiny", d=96, dp=64, T=19)):
        data = P.inputs(spec)
        X, W = P.to_dev(data["X"], "bf16"), P.to_dev(data["W"], "bf16")
        y = ttq.ttq_linear_forward(X, W, None, None, spec.p, spec.lam, spec.alpha, spec.bits,
                                   spec.group, ws=ws, y_dtype=torch.float32)
        y_fresh = ttq.ttq_linear_forward(X, W, None, None, spec.p, spec.lam, spec.alpha,
                                         spec.bits, spec.group, y_dtype=torch.float32)
        torch.cuda.synchronize()
        st, flags = ttq.ttq_get_status(ws)
        assert st == ttq.TTQ_OK, flags
        assert torch.equal(y, y_fresh), spec.name
        outs.append(y)
    assert torch.equal(outs[0], outs[2])


def test_forward_kernel_count_matches_launches():
    """ttq_linear_forward_kernels tells how many kernels a forward call
    enqueues; a CUDA activity trace of one call sees exactly that many of the
    library's kernels (the statistic fused with the scaling of X where the
    rows fit in registers, two kernels where they do not)."""
    from torch.autograd import DeviceType
    from torch.profiler import ProfilerActivity, profile

    cases = [(synth.C2, 3, True),
             # few output tiles: statistic, quantiser, the product split
             # along K and the reduction of its splits
             (synth.C2.with_(dp=512), 4, True),
             (_spec("split_product", d=4096, dp=200, T=333), 4, True),
             # two statistic kernels; 64 rows of W against 4096 tokens and
             # 8192 channels: the product splits along K, then its reduction
             (_spec("long_two_kernel", d=8192, dp=64, T=4096), 5, False),
             (_spec("f32_lowrank", d=448, dp=96, T=77, dtype="f32", r=16), 6, True),
             (_spec("no_tokens", d=512, dp=64, T=0), 2, True),
             # a few tokens: statistic, then the single-pass product
             (_spec("decode", d=1024, dp=640, T=1, bits=4, group=128), 2, True),
             # with a low-rank pair whose A X is split along d: A X, its
             # reduction, then the single-pass product
             (_spec("decode_lowrank", d=8192, dp=256, T=3, bits=2, group=64, r=64), 4, True)]
    for spec, expected, fused in cases:
        data = P.inputs(spec)
        X, W = P.to_dev(data["X"], spec.dtype), P.to_dev(data["W"], spec.dtype)
        A = P.to_dev(data["A"], spec.dtype) if spec.r else None
        B = P.to_dev(data["B"], spec.dtype) if spec.r else None
        ws = ttq.new_workspace(spec.d, spec.dp, spec.T, spec.r, spec.bits, spec.group, _dt(spec))
        n = ttq.ttq_linear_forward_kernels(spec.d, spec.dp, spec.T, spec.r, spec.p, _dt(spec),
                                           spec.bits, spec.group)
        assert n == expected, spec.name
        torch.cuda.synchronize()
        with profile(activities=[ProfilerActivity.CUDA]) as prof:
            ttq.ttq_linear_forward(X, W, A, B, spec.p, spec.lam, spec.alpha, spec.bits, spec.group,
                                   ws=ws, y_dtype=torch.float32)
            torch.cuda.synchronize()
        names = [e.name for e in prof.events() if e.device_type == DeviceType.CUDA]
        ours = [nm for nm in names if "ttq::" in nm]
        assert len(ours) == n, (spec.name, ours)
        assert any("act_norm_scale_kernel" in nm for nm in ours) == fused, (spec.name, ours)
