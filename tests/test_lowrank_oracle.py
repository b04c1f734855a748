"""Pins of the low-rank initialisation oracle (oracle/lowrank.py).

The expected values come from the construction W = U diag(sigma) V^T with
known orthonormal U, V and singular values sigma (the seeded generator
module), not from any SVD: the Eckart-Young closed form of the residual,
the spectral norm of the residual, the best rank-r product itself,
orthonormal rows of A, B = W A^T, the rank-0 and full-rank cases, a
hand-computed 2 x 2 case, and invariance under orthogonal transforms.  A
copy of the oracle with a planted mistake must fail at least one pin.
"""
import os
import sys

import numpy as np
import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
sys.path[:0] = [os.path.join(ROOT, "oracle"), ROOT]

import lowrank  # noqa: E402
from test_weight_quantization_ttq_b200 import synth  # noqa: E402


def _case(dp=48, d=40, m=24, r=6, seed=3):
    sig = synth.geometric_spectrum(m, top=3.0, ratio=0.85, gap_at=r, gap=4.0)
    return synth.spectral_weight(dp, d, sig, seed), r


def check_eckart_young(mod):
    case, r = _case()
    _, _, R = mod.lowrank_init(case["W"], r)
    want = float(np.sum(case["sigma"][r:] ** 2))
    got = float(np.sum(R * R))
    assert abs(got - want) <= 1e-10 * max(1.0, want), (got, want)


def check_spectral_norm(mod):
    case, r = _case(seed=4)
    _, _, R = mod.lowrank_init(case["W"], r)
    assert abs(np.linalg.norm(R, 2) - case["sigma"][r]) <= 1e-10


def check_best_product(mod):
    case, r = _case(seed=5)
    B, A, _ = mod.lowrank_init(case["W"], r)
    U, V, s = case["U"], case["V"], case["sigma"]
    want = (U[:, :r] * s[:r]) @ V[:, :r].T
    assert np.max(np.abs(B @ A - want)) <= 1e-10


def check_factor_shapes_and_split(mod):
    case, r = _case(dp=30, d=50, seed=6)
    B, A, _ = mod.lowrank_init(case["W"], r)
    assert B.shape == (30, r) and A.shape == (r, 50)
    assert np.max(np.abs(A @ A.T - np.eye(r))) <= 1e-12        # orthonormal rows
    assert np.max(np.abs(B - case["W"] @ A.T)) <= 1e-10        # B = W A^T
    # descending: the column norms of B are the singular values
    assert np.allclose(np.linalg.norm(B, axis=0), case["sigma"][:r], rtol=0, atol=1e-10)


def check_rank_edges(mod):
    case, _ = _case(m=12, seed=7)
    W = case["W"]
    B, A, R = mod.lowrank_init(W, 0)
    assert B.shape == (W.shape[0], 0) and A.shape == (0, W.shape[1])
    assert np.array_equal(R, W)
    _, _, R = mod.lowrank_init(W, 12)                            # rank(W) = 12
    assert np.max(np.abs(R)) <= 1e-12


def check_hand_2x2(mod):
    # W = [[3, 0], [0, 1]]: the rank-1 product keeps the 3, the residual is
    # the 1, by hand
    W = np.array([[3.0, 0.0], [0.0, 1.0]])
    B, A, R = mod.lowrank_init(W, 1)
    assert np.allclose(B @ A, [[3.0, 0.0], [0.0, 0.0]], atol=1e-14)
    assert np.allclose(R, [[0.0, 0.0], [0.0, 1.0]], atol=1e-14)


def check_orthogonal_invariance(mod):
    case, r = _case(dp=20, d=16, m=16, seed=8)
    W = case["W"]
    P = synth.orthonormal_columns(20, 20, 101)
    Q = synth.orthonormal_columns(16, 16, 102)
    B, A, _ = mod.lowrank_init(W, r)
    B2, A2, _ = mod.lowrank_init(P @ W @ Q, r)
    assert np.max(np.abs(B2 @ A2 - P @ (B @ A) @ Q)) <= 1e-10


def check_residual_helper(mod):
    case, r = _case(seed=9)
    B, A, R = mod.lowrank_init(case["W"], r)
    assert np.max(np.abs(mod.residual(case["W"], B, A) - R)) <= 1e-14


ALL_CHECKS = [check_eckart_young, check_spectral_norm, check_best_product, check_factor_shapes_and_split,
              check_rank_edges, check_hand_2x2, check_orthogonal_invariance, check_residual_helper]


@pytest.mark.parametrize("chk", ALL_CHECKS, ids=lambda c: c.__name__)
def test_oracle_pin(chk):
    chk(lowrank)


MUTANTS = [
    ("A_from_columns_of_Vt", "A = Vt[:r, :]", "A = Vt[:, :r].T"),
    ("singular_values_dropped", "B = U[:, :r] * S[:r]", "B = U[:, :r]"),
    ("smallest_triplets", "B = U[:, :r] * S[:r]\n    A = Vt[:r, :]", "B = U[:, U.shape[1] - r:] * S[S.size - r:]\n    A = Vt[Vt.shape[0] - r:, :]"),
    ("residual_sign", "return B, A, W64 - B @ A", "return B, A, W64 + B @ A"),
    ("squared_singular_values", "B = U[:, :r] * S[:r]", "B = U[:, :r] * S[:r] ** 2"),
    ("B_transposed_factor", "B = U[:, :r] * S[:r]", "B = (Vt[:r, :].T * S[:r])[:U.shape[0]] if Vt.shape[1] >= U.shape[0] else U[:, :r] * 0"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_is_caught(name, old, new):
    src = open(lowrank.__file__).read()
    assert src.count(old) == 1, name
    ns = {"__name__": "lowrank_mutant"}
    exec(compile(src.replace(old, new), "lowrank_mutant", "exec"), ns)

    class M:
        pass

    mod = M()
    for k in ("lowrank_init", "residual", "singular_values"):
        setattr(mod, k, ns[k])
    failed = []
    for chk in ALL_CHECKS:
        try:
            chk(mod)
        except Exception:
            failed.append(chk.__name__)
    assert failed, f"mutant {name} passed every pin"
