"""The static low-rank initialisation on the GPU (ttq_lowrank_init) against
the oracle (oracle/lowrank.py) and against closed forms.

The GPU computes a randomised truncated SVD, so B A is compared with the
oracle's exact best rank-r product (unique when sigma_r > sigma_{r+1});
B and A themselves are checked for what makes them valid: orthonormal rows
of A and B = W A^T.  W_res must equal W - B A for the B, A the call
returned.  Weights with a known spectrum (seeded orthonormal factors) give
the Eckart-Young residual in closed form, which is also how the full-size
case (d' = 28672, d = 8192, r = 64: the 70B-like MLP shape) is checked
without a CPU SVD of that size.
"""
import numpy as np
import pytest
import torch

import lowrank
import ttq_oracle
from test_weight_quantization_ttq_b200 import synth
from test_weight_quantization_ttq_b200 import ttq

pytestmark = pytest.mark.gpu


def _weight(dp, d, r, m, seed, top=2.0, ratio=0.85, gap=4.0):
    sig = synth.geometric_spectrum(m, top=top, ratio=ratio, gap_at=r, gap=gap)
    return synth.spectral_weight(dp, d, sig, seed)


def _run(W32, r, over, q, dtype, seed=11):
    dp, d = W32.shape
    Om = torch.from_numpy(synth.gaussian_test_matrix(d, r + over, seed)).cuda()
    Wd = torch.from_numpy(np.ascontiguousarray(W32, dtype=np.float32)).to(dtype).cuda()
    n = ttq.ttq_lowrank_workspace_size(dp, d, r, over)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    ttq.ttq_workspace_init(ws)
    B, A, R = ttq.ttq_lowrank_init(Wd, r, Om, power_iters=q, ws=ws)
    torch.cuda.synchronize()
    st, flags = ttq.ttq_get_status(ws)
    return Wd, B, A, R, st, flags, Om, ws


CASES = [
    # d', d, r, oversample, power iterations, modes in W, tolerance on B A
    (300, 200, 16, 8, 2, 80, 1e-4),
    (150, 333, 13, 4, 2, 100, 1e-4),   # l = 17: odd, one idle slot in the Jacobi rounds
    (97, 64, 8, 0, 3, 64, 2e-2),       # no oversampling
    (64, 530, 40, 16, 1, 64, 1e-3),    # d' = l + 8, a wide W
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "dp{}_d{}_r{}_p{}_q{}".format(*c[:5]))
def test_lowrank_f32_matches_oracle(case):
    dp, d, r, over, q, m, tol = case
    c = _weight(dp, d, r, m, seed=dp + d)
    W = c["W"].astype(np.float32)
    Wd, B, A, R, st, flags, Om, _ = _run(W, r, over, q, torch.float32)
    assert st == ttq.TTQ_OK, flags
    Bg = B.cpu().numpy().astype(np.float64)
    Ag = A.cpu().numpy().astype(np.float64)
    Rg = R.cpu().numpy().astype(np.float64)
    W64 = W.astype(np.float64)
    Bo, Ao, Ro = lowrank.lowrank_init(W64, r)
    nW = np.linalg.norm(W64)
    assert np.linalg.norm(Bg @ Ag - Bo @ Ao) / nW <= tol
    assert np.max(np.abs(Ag @ Ag.T - np.eye(r))) <= 1e-4 + 10 * tol
    assert np.linalg.norm(Bg - W64 @ Ag.T) / nW <= 1e-4 + 10 * tol
    # the residual is W - B A for the returned factors, to fp32 rounding
    assert np.max(np.abs(Rg - (W64 - Bg @ Ag))) <= 1e-5 * np.max(np.abs(W64))
    # Eckart-Young: ||W - B A||_F^2 against the closed form sum_{i>r} sigma_i^2
    want = float(np.sum(c["sigma"][r:] ** 2))
    assert abs(float(np.sum(Rg * Rg)) - want) <= max(1e-3, 20 * tol) * want


def test_lowrank_bf16_matches_oracle():
    dp, d, r, over, q = 600, 512, 32, 8, 2
    c = _weight(dp, d, r, 160, seed=21, top=4.0, ratio=0.9, gap=5.0)
    W = synth.bf16_round(c["W"].astype(np.float32))
    Wd, B, A, R, st, flags, Om, _ = _run(W, r, over, q, torch.bfloat16)
    assert st == ttq.TTQ_OK, flags
    assert B.dtype == torch.bfloat16 and A.dtype == torch.bfloat16 and R.dtype == torch.bfloat16
    Bg = B.float().cpu().numpy().astype(np.float64)
    Ag = A.float().cpu().numpy().astype(np.float64)
    Rg = R.float().cpu().numpy().astype(np.float64)
    W64 = W.astype(np.float64)
    Bo, Ao, _ = lowrank.lowrank_init(W64, r)
    nW = np.linalg.norm(W64)
    # B and A are stored in bf16 (8 significant bits)
    assert np.linalg.norm(Bg @ Ag - Bo @ Ao) / nW <= 1e-2
    assert np.max(np.abs(Ag @ Ag.T - np.eye(r))) <= 2e-2
    # W_res is the bf16 rounding (half an ulp: 2^-9 relative) of W - acc,
    # where acc = B A accumulates r exact products in fp32 (error at most
    # r 2^-24 sum_k |B_ik A_kj|); the bound below doubles both terms
    ref = W64 - Bg @ Ag
    bound = 2.0 ** -8 * np.abs(ref) + 2.0 * r * 2.0 ** -24 * (np.abs(Bg) @ np.abs(Ag))
    assert np.all(np.abs(Rg - ref) <= bound)


def test_lowrank_deterministic_and_residual_optional():
    c = _weight(200, 160, 12, 60, seed=3)
    W = c["W"].astype(np.float32)
    Wd, B1, A1, R1, st, _, Om, ws = _run(W, 12, 8, 2, torch.float32)
    B2, A2, R2 = ttq.ttq_lowrank_init(Wd, 12, Om, power_iters=2, ws=ws)
    B3, A3, R3 = ttq.ttq_lowrank_init(Wd, 12, Om, power_iters=2, ws=ws, residual=False)
    torch.cuda.synchronize()
    assert R3 is None
    assert torch.equal(B1, B2) and torch.equal(A1, A2) and torch.equal(R1, R2)
    assert torch.equal(B1, B3) and torch.equal(A1, A3)


def test_lowrank_zero_weight_is_flagged_and_finite():
    W = np.zeros((128, 96), dtype=np.float32)
    Wd, B, A, R, st, flags, _, _ = _run(W, 8, 8, 1, torch.float32)
    assert flags & ttq.TTQ_FLAG_RANK_DEFICIENT
    assert st == ttq.TTQ_OK, flags          # rank deficiency is a warning
    assert not flags & ttq.TTQ_FLAG_NONFINITE
    assert torch.count_nonzero(B) == 0 and torch.count_nonzero(A) == 0 and torch.count_nonzero(R) == 0


def test_lowrank_then_forward_matches_oracle():
    # the residual and the factors go into the layer; the forward equals
    # the oracle's forward on the same W_res, A, B
    spec = synth.LinearSpec("lowrank_fwd", d=512, dp=384, T=40, bits=2, group=64, r=24,
                            n_outliers=6, outlier_lo=20.0, outlier_hi=60.0)
    data = synth.generate(spec, need_w=False)
    c = _weight(384, 512, 24, 200, seed=5, top=8.0, ratio=0.97, gap=1.0)
    W = synth.bf16_round(c["W"].astype(np.float32))
    Wd, B, A, R, st, flags, _, _ = _run(W, 24, 8, 2, torch.bfloat16)
    assert st == ttq.TTQ_OK, flags
    X = torch.from_numpy(data["X"]).to(torch.bfloat16).cuda()
    Y = ttq.ttq_linear_forward(X, R, A, B, spec.p, spec.lam, spec.alpha, spec.bits, spec.group,
                               y_dtype=torch.float32)
    torch.cuda.synchronize()
    O = ttq_oracle.get()
    ref = O.forward(data["X"].astype(np.float64), R.float().cpu().numpy(), spec.p, spec.lam, spec.alpha,
                    spec.bits, spec.group, A=A.float().cpu().numpy(), B=B.float().cpu().numpy())
    Yr = ref["Y"]
    err = float(np.max(np.abs(Y.cpu().numpy() - Yr))) / float(np.sqrt(np.mean(Yr ** 2)))
    assert err <= 1e-2, err


def test_lowrank_full_size_closed_form():
    # the 70B-like MLP shape: d' = 28672, d = 8192, r = 64, bf16; W has 128
    # modes with a gap after 64
    dp, d, r, over, q = 28672, 8192, 64, 8, 2
    sig = synth.geometric_spectrum(128, top=40.0, ratio=0.97, gap_at=r, gap=3.0)
    c = synth.spectral_weight(dp, d, sig, seed=1)
    W32 = c["W"].astype(np.float32)
    W = synth.bf16_round(W32)
    E = W.astype(np.float64) - c["W"]                      # the bf16 rounding of W
    Wd, B, A, R, st, flags, _, _ = _run(W, r, over, q, torch.bfloat16)
    assert st == ttq.TTQ_OK, flags
    Rg = R.float()
    res2 = float(torch.sum(Rg.double() ** 2).cpu())
    want = float(np.sum(sig[r:] ** 2)) + float(np.sum(E * E))
    assert abs(res2 - want) <= 2e-2 * want, (res2, want)
    # sampled rows of B A against the construction's best rank-r product
    rows = synth.sample_rows(dp, 64)
    BA = (B.float()[torch.from_numpy(rows).cuda()] @ A.float()).double().cpu().numpy()
    U, V = c["U"], c["V"]
    BAo = (U[rows, :r] * sig[:r]) @ V[:, :r].T
    Wrow = np.linalg.norm(c["W"][rows], axis=1)
    assert np.max(np.linalg.norm(BA - BAo, axis=1) / Wrow) <= 2e-2
    Ag = A.float()
    assert float(torch.max(torch.abs(Ag @ Ag.T - torch.eye(r, device="cuda")))) <= 2e-2
