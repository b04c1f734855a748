"""Static low-rank initialisation of the TTQ layer, CPU oracle.

TEST INFRASTRUCTURE ONLY.  Only the test suite, the package smoke check and
the benchmark's CPU-baseline / reference leg may import this module; the
product path never does.  It shares no code with the CUDA library.

The pages decompose the weight as W ~ W_q + B A, with B, A static factors
initialised by PCA and W_q the quantised residual (gist.science/zh/paper/
2603.19296, section 2.2; gist.science/nl/paper/2603.19296, section 2
"Kerncomponenten", item 3).  Readings taken here:
- "PCA of W" is the truncated singular value decomposition of W itself,
  without centring: the rank-r product B A that leaves the smallest
  residual W - B A (Eckart-Young) is U_r S_r V_r^T, and a centred PCA would
  not reproduce W.
- The split between the factors: B = U_r S_r (d' x r), A = V_r^T (r x d),
  so the rows of A are orthonormal principal directions of the input space
  and B holds each output row's coordinates along them (B = W A^T).
- The residual fed to the quantiser is W - B A with B and A as stored
  (rounded to the layer's dtype, when it is bf16).
The decomposition is LAPACK's (numpy.linalg.svd) in float64.
"""
from __future__ import annotations

import numpy as np


def lowrank_init(W: np.ndarray, r: int) -> tuple[np.ndarray, np.ndarray, np.ndarray]:
    """(B [d'][r], A [r][d], W - B A [d'][d]), all float64, for the rank-r
    truncated SVD of W [d'][d]."""
    W64 = np.asarray(W, dtype=np.float64)
    dp, d = W64.shape
    if not 0 <= r <= min(dp, d):
        raise ValueError("rank out of range")
    U, S, Vt = np.linalg.svd(W64, full_matrices=False)
    B = U[:, :r] * S[:r]
    A = Vt[:r, :]
    return B, A, W64 - B @ A


def residual(W: np.ndarray, B: np.ndarray, A: np.ndarray) -> np.ndarray:
    """W - B A in float64 for given factors."""
    return np.asarray(W, np.float64) - np.asarray(B, np.float64) @ np.asarray(A, np.float64)


def singular_values(W: np.ndarray) -> np.ndarray:
    """The singular values of W, descending (float64)."""
    return np.linalg.svd(np.asarray(W, np.float64), compute_uv=False)
