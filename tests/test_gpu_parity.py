"""CUDA path vs the CPU oracle, element by element, through the C ABI.

Sizes: small and ragged shapes that span several tiles with a tail, and the
five workloads at full size (sampled output rows for Y; D and the codes,
scales and zeros always in full).
"""
import numpy as np
import pytest
import torch

import parity as P
import ttq_oracle
from test_weight_quantization_ttq_b200 import synth
from test_weight_quantization_ttq_b200 import ttq

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def O():
    return ttq_oracle.get()


def _small(name, d, dp, T, bits, group, dtype="bf16", r=0, p=2.0, lam=1e-3, alpha=0.5, n_out=3, seed=0):
    return synth.LinearSpec(name, d=d, dp=dp, T=T, bits=bits, group=group, dtype=dtype, r=r, p=p,
                            lam=lam, alpha=alpha, n_outliers=n_out, outlier_lo=20.0, outlier_hi=80.0,
                            seed=seed)


ACT_CASES = [
    synth.C1,
    synth.C2,
    synth.C3_DOWN,
    synth.C4.with_(T=1),
    synth.C4.with_(T=16),
    synth.C5.with_(T=4096, p=1.0, alpha=0.25),
    synth.C5.with_(T=128, p=2.0, alpha=0.5),
    _small("p3_ragged", d=264, dp=0, T=45, bits=4, group=8 * 1, p=3.0),
    _small("one_token", d=64, dp=0, T=1, bits=4, group=32),
    _small("f32_many_tokens", d=512, dp=0, T=3000, bits=4, group=32, dtype="f32"),
]


@pytest.mark.parametrize("spec", ACT_CASES, ids=lambda s: f"{s.name}-T{s.T}")
def test_act_norm_matches_oracle(O, spec):
    x = P.inputs(spec, need_w=False)["X"]
    D_ref, Dr_ref, st = O.act_norm(x.astype(np.float64), *P.params(spec))
    assert st == 0
    X = P.to_dev(x, spec.dtype)
    D, Dr = ttq.ttq_act_norm(X, spec.p, spec.lam, spec.alpha)
    torch.cuda.synchronize()
    D, Dr = D.cpu().numpy().astype(np.float64), Dr.cpu().numpy().astype(np.float64)
    assert np.max(np.abs(D - D_ref) / D_ref) <= P.D_RTOL
    assert np.max(np.abs(Dr - Dr_ref) / Dr_ref) <= P.D_RTOL


def test_act_norm_empty_tokens(O):
    d = 96
    X = torch.empty((0, d), dtype=torch.bfloat16, device="cuda")
    D, Dr = ttq.ttq_act_norm(X, 2.0, 0.25, 0.5)
    torch.cuda.synchronize()
    assert np.allclose(D.cpu().numpy(), 0.25 ** 0.5, rtol=1e-7)
    assert np.allclose(Dr.cpu().numpy(), 0.25 ** -0.25, rtol=1e-7)


QUANT_CASES = [
    (synth.C1, None),
    (synth.C2, None),
    (synth.C3_GATE, None),
    (synth.C3_DOWN, None),
    (synth.C4, None),
    (synth.C5, None),
]
for _bits in (2, 3, 4):
    for _g in (32, 64, 128, 256):
        QUANT_CASES.append((_small(f"b{_bits}g{_g}", d=512, dp=37, T=9, bits=_bits, group=_g), None))
QUANT_CASES.append((_small("f32_b3g32_d96", d=96, dp=5, T=4, bits=3, group=32, dtype="f32"), None))
QUANT_CASES.append((_small("identity_D", d=256, dp=64, T=4, bits=4, group=64), "identity"))


@pytest.mark.parametrize("spec,mode", QUANT_CASES, ids=lambda v: getattr(v, "name", str(v)))
def test_quantize_bit_exact(O, spec, mode):
    data = P.inputs(spec)
    W = data["W"]
    if mode == "identity":
        D32 = None
    else:
        D_ref, _, _ = O.act_norm(data["X"].astype(np.float64), *P.params(spec))
        D32 = D_ref.astype(np.float32)  # both sides get this same D
    codes_ref, sc_ref, ze_ref, st = O.quantize(W, D32, spec.bits, spec.group)
    assert st == 0
    Dd = None if D32 is None else torch.from_numpy(D32).cuda()
    codes, sc, ze = ttq.ttq_quantize_weight(P.to_dev(W, spec.dtype), Dd, spec.bits, spec.group)
    torch.cuda.synchronize()
    assert np.array_equal(P.u32(codes), codes_ref)
    assert np.array_equal(P.u16(sc), sc_ref)
    assert np.array_equal(P.u16(ze), ze_ref)


GEMM_CASES = [
    # d, dp, T, bits, group, r, dtype
    (64, 128, 1, 4, 32, 0, "bf16"),
    (96, 200, 7, 3, 32, 0, "bf16"),
    (320, 256, 16, 2, 64, 0, "bf16"),
    (256, 130, 17, 4, 64, 0, "bf16"),
    (512, 384, 100, 4, 128, 0, "bf16"),
    (512, 256, 256, 3, 128, 0, "bf16"),
    (768, 300, 300, 2, 64, 0, "bf16"),
    (1024, 256, 600, 4, 256, 0, "bf16"),
    (256, 256, 64, 4, 64, 0, "f32"),
    (512, 200, 40, 3, 128, 32, "bf16"),
    (512, 256, 300, 2, 64, 8, "bf16"),
    (640, 128, 33, 4, 128, 72, "bf16"),
    (256, 128, 20, 4, 64, 16, "f32"),
    # at most 16 tokens: the register-dequantising product, with K tails of
    # 32 channels, ragged rows and the low-rank term
    (96, 64, 5, 4, 32, 0, "bf16"),
    (512, 200, 9, 4, 64, 16, "bf16"),
    (288, 100, 3, 3, 32, 8, "f32"),
    (352, 70, 16, 2, 32, 24, "bf16"),
    (4096, 333, 2, 4, 128, 64, "bf16"),
    (384, 100, 5, 3, 64, 8, "bf16"),
    (1024, 64, 13, 3, 256, 0, "f32"),
]


@pytest.mark.parametrize("case", GEMM_CASES, ids=lambda c: "d{}_dp{}_T{}_b{}_g{}_r{}_{}".format(*c))
def test_dequant_gemm_matches_oracle(O, case):
    d, dp, T, bits, group, r, dtype = case
    spec = _small("gemm", d=d, dp=dp, T=T, bits=bits, group=group, dtype=dtype, r=r)
    data = P.inputs(spec)
    X = data["X"].astype(np.float64)
    D_ref, Dr_ref, _ = O.act_norm(X, *P.params(spec))
    codes, sc, ze, _ = O.quantize(data["W"], D_ref.astype(np.float32), bits, group)
    Dr32 = Dr_ref.astype(np.float32)
    What = O.dequant_rows(codes, sc, ze, Dr32.astype(np.float64), d, bits, group)
    Y_ref = O.project(What, X)
    if r > 0:
        Y_ref = O.lowrank_add(data["A"], data["B"], X, Y_ref)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    A = P.to_dev(data["A"], dtype) if r > 0 else None
    B = P.to_dev(data["B"], dtype) if r > 0 else None
    args = (dev(codes.view(np.int32)), dev(sc.view(np.int16)), dev(ze.view(np.int16)), dev(Dr32),
            P.to_dev(data["X"], dtype), A, B, bits, group)
    Y = ttq.ttq_dequant_gemm(*args, y_dtype=torch.float32)
    Yb = ttq.ttq_dequant_gemm(*args, y_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    err = P.y_error(Y.cpu().numpy(), Y_ref)
    assert err <= P.Y_TOL, err
    # the bf16 output is the fp32 accumulator rounded once to nearest-even
    assert torch.equal(Yb, Y.to(torch.bfloat16))


# every configured workload point: the fp32 d = 256 layer, the q_proj
# prefill, the three MLP projections, decode at T = 1, 4, 16 and all twenty
# points of the 70B-like MLP shape (T x p x alpha)
FORWARD_CASES = [spec for name in ("C1", "C2", "C3", "C4", "C5") for spec in synth.CONFIGS[name]] + [
    _small("ragged_all", d=96, dp=200, T=19, bits=3, group=32),
    # 256-row tiles with ragged row and token tails
    _small("ragged_256row_tiles", d=4096, dp=4296, T=2000, bits=4, group=128, n_out=40),
    _small("ragged_256row_tiles_int2_lowrank", d=1024, dp=4296, T=2000, bits=2, group=64, r=40, n_out=10),
    _small("ragged_lowrank", d=448, dp=333, T=77, bits=2, group=64, r=24),
    _small("decode_lowrank", d=480, dp=150, T=11, bits=4, group=32, r=16),
    _small("decode_int3_lowrank", d=736, dp=77, T=1, bits=3, group=32, r=8, dtype="f32"),
    _small("decode_int3_k768", d=768, dp=129, T=8, bits=3, group=128, r=16),
    # the product on W_hat split along K (few output tiles, long K): ragged
    # rows, tokens and last K block, and the low-rank tail in the last split
    _small("split_k_ragged_lowrank", d=8224, dp=300, T=333, bits=4, group=32, r=16),
    _small("split_k_int2_lowrank", d=4128, dp=264, T=520, bits=2, group=32, r=24),
    _small("split_k_eight", d=4096, dp=200, T=333, bits=3, group=64),
    # T x d' odd: the split reduction's element-wise path (and Y rows of an
    # odd length)
    _small("split_k_odd_rows_lowrank", d=4096, dp=201, T=333, bits=4, group=32, r=16),
]


@pytest.mark.parametrize("spec", FORWARD_CASES, ids=lambda s: f"{s.name}-T{s.T}-p{s.p}-a{s.alpha}")
def test_forward_matches_oracle(O, spec):
    data = P.inputs_shared_w(spec)
    rows = synth.sample_rows(spec.dp, 96)
    ref = O.forward(data["X"].astype(np.float64), data["W"], *P.params(spec), spec.bits,
                    spec.group, A=data.get("A"), B=data.get("B"), rows=rows)
    assert ref["status"] == 0
    X = P.to_dev(data["X"], spec.dtype)
    W = P.to_dev(data["W"], spec.dtype)
    A = P.to_dev(data["A"], spec.dtype) if spec.r else None
    B = P.to_dev(data["B"], spec.dtype) if spec.r else None
    dt = ttq.TTQ_F32 if spec.dtype == "f32" else ttq.TTQ_BF16
    ws = ttq.new_workspace(spec.d, spec.dp, spec.T, spec.r, spec.bits, spec.group, dt)
    Y = ttq.ttq_linear_forward(X, W, A, B, spec.p, spec.lam, spec.alpha, spec.bits, spec.group, ws=ws,
                               y_dtype=torch.float32)
    Yo = ttq.ttq_linear_forward(X, W, A, B, spec.p, spec.lam, spec.alpha, spec.bits, spec.group, ws=ws,
                                y_dtype=X.dtype)
    torch.cuda.synchronize()
    assert torch.equal(Yo, Y.to(X.dtype))
    st, flags = ttq.ttq_get_status(ws)
    assert st == ttq.TTQ_OK, flags
    views = ttq.workspace_views(ws, spec.d, spec.dp, spec.T, spec.r, spec.bits, spec.group, dt)
    D = views["D"].cpu().numpy().astype(np.float64)
    assert np.max(np.abs(D - ref["D"]) / ref["D"]) <= P.D_RTOL
    codes_dev = views["codes"]
    sc_dev, ze_dev = views["scales"], views["zeros"]
    if "wq" in views:
        # the forward kept the binary16 W_hat and no codes: the quantiser,
        # given the forward's D, gives the codes, and W_hat is their
        # dequantisation to the bit
        codes_dev, sc_dev, ze_dev = ttq.ttq_quantize_weight(W, views["D"], spec.bits, spec.group)
        torch.cuda.synchronize()
        q = O.unpack(P.u32(codes_dev), spec.d, spec.bits).astype(np.float64)
        k = np.arange(spec.d) // spec.group
        sv = P.u16(sc_dev).view(np.float16).astype(np.float64)[:, k]
        zv = P.u16(ze_dev).view(np.float16).astype(np.float64)[:, k]
        assert np.array_equal(views["wq"].cpu().numpy().view(np.uint16),
                              (sv * (q - zv)).astype(np.float16).view(np.uint16))
    elif ttq.ttq_workspace_get_layout(spec.d, spec.dp, spec.T, spec.r, spec.bits, spec.group, dt).tickets:
        # the forward took the single-pass product, which writes no codes: the
        # same kernel, given the forward's own D and X D^(-1/2), stores them on
        # request, and its Y is the forward's to the bit
        codes_dev = torch.empty_like(views["codes"])
        sc_dev, ze_dev = torch.empty_like(views["scales"]), torch.empty_like(views["zeros"])
        Y1 = ttq.ttq_quantize_gemm(W, views["D"], views["xh"], A, B, X if spec.r else None, spec.bits,
                                   spec.group, y_dtype=torch.float32, codes=codes_dev, scales=sc_dev,
                                   zeros=ze_dev)
        torch.cuda.synchronize()
        assert torch.equal(Y1, Y)
    # The quantiser is bit-exact for a shared D (test_quantize_bit_exact); here
    # each side uses its own D, so codes, scales and zeros must agree in every
    # group whose channels got the same binary32 D on both sides.
    same_d = views["D"].cpu().numpy() == ref["D"].astype(np.float32)
    group_ok = same_d.reshape(-1, spec.group).all(axis=1)          # [d/group]
    wpg = spec.group * spec.bits // 32                               # words per group
    codes = P.u32(codes_dev).reshape(spec.dp, -1, wpg)
    ref_codes = ref["codes"].reshape(spec.dp, -1, wpg)
    assert np.array_equal(codes[:, group_ok], ref_codes[:, group_ok])
    assert np.array_equal(P.u16(sc_dev)[:, group_ok], ref["scales"][:, group_ok])
    assert np.array_equal(P.u16(ze_dev)[:, group_ok], ref["zeros"][:, group_ok])
    assert group_ok.mean() >= 0.99, f"D differs in {np.count_nonzero(~same_d)} channels"
    err = P.y_error(Y.cpu().numpy()[:, rows], ref["Y"])
    assert err <= P.Y_TOL, err


def test_scale_activations_rounds_once():
    """X D^{-1/2} in binary16 is the float32 product rounded once."""
    rng = np.random.default_rng(3)
    T, d = 37, 264
    x = P.inputs(_small("scale", d=d, dp=0, T=T, bits=4, group=8), need_w=False)["X"]
    dr = np.exp(rng.uniform(-3, 1, d)).astype(np.float32)
    for dtype in ("bf16", "f32"):
        Xs = ttq.ttq_scale_activations(P.to_dev(x, dtype), torch.from_numpy(dr).cuda())
        torch.cuda.synchronize()
        ref = (x.astype(np.float32) * dr[None, :]).astype(np.float16)
        assert np.array_equal(Xs.cpu().numpy().view(np.uint16), ref.view(np.uint16)), dtype


def test_composed_steps_equal_forward(O):
    """act_norm -> scale_activations -> quantize_weight -> dequant_gemm (binary16
    X D^{-1/2}) is the forward, bit for bit, and matches the oracle.  The
    shape's product on the materialised weight is not split along K (a split
    adds its partial sums in another order than the codes' one-pass product;
    those shapes are checked against the oracle in test_forward_matches_oracle)."""
    spec = synth.C2.with_(T=1024)
    data = P.inputs(spec)
    X, W = P.to_dev(data["X"], "bf16"), P.to_dev(data["W"], "bf16")
    p, lam, alpha = spec.p, spec.lam, spec.alpha
    Y = ttq.ttq_linear_forward(X, W, None, None, p, lam, alpha, spec.bits, spec.group, y_dtype=torch.float32)
    D, Dr = ttq.ttq_act_norm(X, p, lam, alpha)
    Xs = ttq.ttq_scale_activations(X, Dr)
    codes, sc, ze = ttq.ttq_quantize_weight(W, D, spec.bits, spec.group)
    Y2 = ttq.ttq_dequant_gemm(codes, sc, ze, None, Xs, None, None, spec.bits, spec.group,
                              y_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(Y, Y2)
    rows = synth.sample_rows(spec.dp, 64)
    ref = O.forward(data["X"].astype(np.float64), data["W"], *P.params(spec), spec.bits, spec.group, rows=rows)
    assert P.y_error(Y2.cpu().numpy()[:, rows], ref["Y"]) <= P.Y_TOL


def test_forward_is_deterministic():
    spec = synth.C2.with_(T=300)
    data = P.inputs(spec)
    X, W = P.to_dev(data["X"], "bf16"), P.to_dev(data["W"], "bf16")
    y1 = ttq.ttq_linear_forward(X, W, None, None, spec.p, spec.lam, spec.alpha, spec.bits, spec.group)
    y2 = ttq.ttq_linear_forward(X, W, None, None, spec.p, spec.lam, spec.alpha, spec.bits, spec.group)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)


def test_forward_empty_tokens():
    d, dp = 128, 64
    X = torch.empty((0, d), dtype=torch.bfloat16, device="cuda")
    W = torch.randn((dp, d), device="cuda").to(torch.bfloat16)
    Y = ttq.ttq_linear_forward(X, W, None, None, 2.0, 1e-3, 0.5, 4, 64)
    torch.cuda.synchronize()
    assert Y.shape == (0, dp)


def test_status_flags_nonfinite():
    d, dp, T = 128, 64, 8
    X = torch.randn((T, d), device="cuda").to(torch.bfloat16)
    W = torch.randn((dp, d), device="cuda").to(torch.bfloat16)
    X[3, 5] = float("nan")
    ws = ttq.new_workspace(d, dp, T, 0, 4, 64)
    ttq.ttq_linear_forward(X, W, None, None, 2.0, 1e-3, 0.5, 4, 64, ws=ws)
    torch.cuda.synchronize()
    st, flags = ttq.ttq_get_status(ws)
    assert st == ttq.TTQ_ERR_NONFINITE and flags & ttq.TTQ_FLAG_NONFINITE
    # lambda = 0 and an all-zero channel: D_ii = 0
    X2 = torch.randn((T, d), device="cuda").to(torch.bfloat16)
    X2[:, 7] = 0
    ttq.ttq_workspace_init(ws)
    ttq.ttq_linear_forward(X2, W, None, None, 2.0, 0.0, 0.5, 4, 64, ws=ws)
    torch.cuda.synchronize()
    assert ttq.ttq_get_status(ws)[0] == ttq.TTQ_ERR_NONFINITE
    # a group whose binary16 scale overflows
    W2 = W.clone()
    W2[0, 0] = 3.0e6
    ttq.ttq_workspace_init(ws)
    ttq.ttq_quantize_weight(W2, None, 4, 64, ws=ws)
    torch.cuda.synchronize()
    st, flags = ttq.ttq_get_status(ws)
    assert st == ttq.TTQ_ERR_NONFINITE and flags & ttq.TTQ_FLAG_SCALE_OVERFLOW
    # X D^{-1/2} beyond the binary16 range of the product's operand (alpha = 0
    # gives D = I; with alpha > 0 the outlier's own norm would shrink it)
    X3 = X2 + 1
    X3[2, 9] = 1.0e5
    ttq.ttq_workspace_init(ws)
    ttq.ttq_linear_forward(X3, W, None, None, 2.0, 1e-3, 0.0, 4, 64, ws=ws)
    torch.cuda.synchronize()
    st, flags = ttq.ttq_get_status(ws)
    assert st == ttq.TTQ_ERR_NONFINITE and flags & ttq.TTQ_FLAG_X_RANGE
    # and a clean call after a reset reads OK
    ttq.ttq_workspace_init(ws)
    ttq.ttq_linear_forward(X2 + 1, W, None, None, 2.0, 1e-3, 0.5, 4, 64, ws=ws)
    torch.cuda.synchronize()
    assert ttq.ttq_get_status(ws)[0] == ttq.TTQ_OK


def test_invalid_arguments_are_rejected():
    X = torch.randn((4, 128), device="cuda").to(torch.bfloat16)
    W = torch.randn((64, 128), device="cuda").to(torch.bfloat16)
    with pytest.raises(ttq.TTQError) as e:
        ttq.ttq_linear_forward(X, W, None, None, 0.5, 1e-3, 0.5, 4, 64)  # p < 1
    assert e.value.status == ttq.TTQ_ERR_INVALID_ARG
    with pytest.raises(ttq.TTQError) as e:
        ttq.ttq_quantize_weight(W, None, 5, 64)
    assert e.value.status == ttq.TTQ_ERR_UNSUPPORTED
    ws = torch.empty(1024, dtype=torch.uint8, device="cuda")
    with pytest.raises(ttq.TTQError) as e:
        ttq.ttq_linear_forward(X, W, None, None, 2.0, 1e-3, 0.5, 4, 64, ws=ws)
    assert e.value.status == ttq.TTQ_ERR_WORKSPACE
