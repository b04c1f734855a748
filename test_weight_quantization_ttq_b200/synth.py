"""Seeded synthetic inputs for the TTQ linear layer.

This module only draws random tensors; it holds none of the method's
arithmetic, and it is the one piece shared by the CUDA path's tests/bench and
the CPU oracle.  The pages measure on WikiText-2, PTB, C4, TextVQA and
LIBERO with trained OPT/Qwen3/Gemma3 checkpoints (gist.science/zh/paper/
2603.19296, section 4); none of that is available, so these seeded tensors
stand in for the activations and weights, with the outlier-channel
structure the pages describe (a few input channels 10-100x larger than the
rest: blog.lo0.es "Test-time quantization", TL;DR).

Recipe: ``numpy.random.Generator(PCG64)`` seeded from ``SeedSequence(seed)``
spawned into six child streams, used in this fixed order: X, W, A, B, the
outlier-channel choice, the outlier factors.  Values are drawn in float32
and, for bf16 layers, rounded to bfloat16 (round-to-nearest-even); the
returned float32 arrays hold exactly the values the device receives.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import numpy as np


def bf16_round(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); the
    result is returned as float32 holding bf16-representable values."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32)
    # finite inputs cannot carry past bit 31: the largest is 0xFF7FFFFF + 0x8000
    u = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) & np.uint32(0xFFFF0000)
    return u.view(np.float32).reshape(a.shape)


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """The uint16 bit patterns of bf16-representable float32 values."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    return (a.view(np.uint32) >> 16).astype(np.uint16)


@dataclass(frozen=True)
class LinearSpec:
    """One TTQ linear call: shapes, quantiser and statistic parameters, and
    the distribution recipe of its inputs."""

    name: str
    d: int                 # input channels
    dp: int                # output channels d'
    T: int                 # tokens
    bits: int
    group: int
    p: float = 2.0
    lam: float = 1e-3
    alpha: float = 0.5
    r: int = 0             # low-rank rank (0: no B(AX) term)
    dtype: str = "bf16"    # "bf16" or "f32" for X, W, A, B and Y
    w_std: float = 0.02
    ab_std: float = 0.01
    n_outliers: int = 0
    outlier_lo: float = 50.0   # outlier factor, log-uniform in [lo, hi]
    outlier_hi: float = 50.0
    x_kind: str = "normal"     # "normal" or "silu_gated"
    seed: int = 0

    def with_(self, **kw) -> "LinearSpec":
        return replace(self, **kw)


# The five workloads.  Sizes, bit widths, groups and distributions follow the
# layer shapes the pages discuss (LLM projections at 4096 and 8192 width,
# decode and prefill token counts, INT2-INT4 with and without a static
# low-rank term).
C1 = LinearSpec("ttq_linear_fp32_d256", d=256, dp=256, T=64, bits=4, group=64,
                dtype="f32", w_std=1.0 / 16.0, n_outliers=4)
C2 = LinearSpec("q_proj_prefill_4096", d=4096, dp=4096, T=2048, bits=4, group=128,
                n_outliers=40, outlier_lo=20.0, outlier_hi=100.0)
C3_GATE = LinearSpec("mlp_gate_4096x11008", d=4096, dp=11008, T=512, bits=3, group=128,
                     r=32, n_outliers=4, seed=0)
C3_UP = C3_GATE.with_(name="mlp_up_4096x11008", seed=1)
C3_DOWN = LinearSpec("mlp_down_11008x4096", d=11008, dp=4096, T=512, bits=3, group=128,
                     r=32, n_outliers=4, x_kind="silu_gated", seed=2)
C4 = LinearSpec("decode_4096x14336", d=4096, dp=14336, T=1, bits=4, group=128,
                n_outliers=40)
C4_TOKENS = (1, 4, 16)
C5 = LinearSpec("mlp70b_8192x28672", d=8192, dp=28672, T=1, bits=2, group=64, r=64,
                w_std=0.015, n_outliers=40, outlier_lo=10.0, outlier_hi=100.0)
C5_TOKENS = (1, 16, 128, 1024, 4096)
C5_P = (1.0, 2.0)
C5_ALPHA = (0.25, 0.5)

CONFIGS = {
    "C1": [C1],
    "C2": [C2],
    "C3": [C3_GATE, C3_UP, C3_DOWN],
    "C4": [C4.with_(T=t) for t in C4_TOKENS],
    "C5": [C5.with_(T=t, p=p, alpha=a) for t in C5_TOKENS for p in C5_P for a in C5_ALPHA],
}


def _streams(seed: int):
    ss = np.random.SeedSequence(seed)
    return [np.random.Generator(np.random.PCG64(c)) for c in ss.spawn(6)]


def generate(spec: LinearSpec, rows: np.ndarray | None = None, need_w: bool = True) -> dict:
    """Draw X [T][d], W [d'][d], A [r][d], B [d'][r] for one spec.

    ``rows`` is unused by the draw itself (W is always drawn whole so that
    every caller sees the same tensor); ``need_w=False`` skips W for callers
    that only need activations.
    """
    del rows
    gx, gw, ga, gb, gc, gf = _streams(spec.seed)
    T, d, dp = spec.T, spec.d, spec.dp
    if spec.x_kind == "silu_gated":
        u = gx.standard_normal((T, d), dtype=np.float32)
        v = gx.standard_normal((T, d), dtype=np.float32)
        X = (u / (1.0 + np.exp(-u))) * v  # SiLU(u) * v: a gated MLP hidden state
    else:
        X = gx.standard_normal((T, d), dtype=np.float32)
    if spec.n_outliers > 0:
        ch = gc.choice(d, size=spec.n_outliers, replace=False)
        if spec.outlier_hi > spec.outlier_lo:
            f = np.exp(gf.uniform(np.log(spec.outlier_lo), np.log(spec.outlier_hi),
                                  size=spec.n_outliers)).astype(np.float32)
        else:
            f = np.full(spec.n_outliers, spec.outlier_lo, np.float32)
        X[:, ch] *= f[None, :]
    else:
        ch = np.zeros(0, np.int64)
    out = {"spec": spec, "outlier_channels": np.sort(ch)}
    rnd = (lambda a: bf16_round(a)) if spec.dtype == "bf16" else (lambda a: np.ascontiguousarray(a, np.float32))
    out["X"] = rnd(X)
    if need_w:
        out["W"] = rnd(gw.standard_normal((dp, d), dtype=np.float32) * np.float32(spec.w_std))
    if spec.r > 0:
        out["A"] = rnd(ga.standard_normal((spec.r, d), dtype=np.float32) * np.float32(spec.ab_std))
        out["B"] = rnd(gb.standard_normal((dp, spec.r), dtype=np.float32) * np.float32(spec.ab_std))
    return out


def sample_rows(dp: int, n: int, seed: int = 12345) -> np.ndarray:
    """A seeded, sorted sample of output rows, always including the first
    and the last row (the ragged tile edges)."""
    g = np.random.Generator(np.random.PCG64(seed))
    n = min(n, dp)
    picked = set(g.choice(dp, size=max(0, n - 2), replace=False).tolist()) | {0, dp - 1}
    return np.array(sorted(picked), dtype=np.int64)


# ------------------------------------------------------- low-rank structure
# Inputs for the static low-rank initialisation (B, A from W): a weight with
# a known spectrum, and the Gaussian test matrix a randomised range finder
# draws.  Both are drawn here so that the CUDA path and the oracle see the
# same values; nothing below computes any part of the method.

def orthonormal_columns(n: int, m: int, seed: int) -> np.ndarray:
    """n x m float64 with orthonormal columns (Q of a seeded Gaussian, its
    column signs fixed so that diag(R) > 0)."""
    g = np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed)))
    q, rr = np.linalg.qr(g.standard_normal((n, m)))
    return q * np.where(np.diag(rr) < 0, -1.0, 1.0)


def spectral_weight(dp: int, d: int, sigma: np.ndarray, seed: int = 0) -> dict:
    """W = U diag(sigma) V^T (float64, d' x d) from seeded orthonormal U
    (d' x m) and V (d x m), m = len(sigma); returns W, U, V and sigma so that
    a test knows W's singular triplets without computing them."""
    sigma = np.asarray(sigma, dtype=np.float64)
    m = sigma.size
    U = orthonormal_columns(dp, m, seed * 2 + 1)
    V = orthonormal_columns(d, m, seed * 2 + 2)
    return {"W": (U * sigma) @ V.T, "U": U, "V": V, "sigma": sigma}


def geometric_spectrum(m: int, top: float = 1.0, ratio: float = 0.9, gap_at: int = 0,
                       gap: float = 1.0) -> np.ndarray:
    """sigma_i = top * ratio^i, i < m, divided by `gap` from index gap_at on
    (a spectral gap after the first gap_at values when gap > 1)."""
    s = top * ratio ** np.arange(m, dtype=np.float64)
    if gap_at > 0:
        s[gap_at:] /= gap
    return s


def gaussian_test_matrix(d: int, l: int, seed: int = 7) -> np.ndarray:
    """d x l float32 standard normal draws (the range finder's test matrix)."""
    g = np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed)))
    return g.standard_normal((d, l), dtype=np.float32)
