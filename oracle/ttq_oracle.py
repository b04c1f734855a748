"""numpy front end of the TTQ CPU oracle (``ttq_oracle.c``).

TEST INFRASTRUCTURE ONLY.  Only the test suite, the package smoke check and
the benchmark's CPU-baseline / reference leg may import this module; the
product path never does.  The oracle shares no code with the CUDA library.

Each function follows one step of the method as the pages state it
(arXiv:2603.19296 as summarised on gist.science/zh/paper/2603.19296,
sections 2.1-2.3, and the affine quantiser of the blog.lo0.es post
"Test-time quantization ...", section "The maths that matter"); the C file
documents the readings taken where the pages are silent.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import tempfile

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "ttq_oracle.c")
LIBRARY = os.path.join(_HERE, "libttq_oracle.so")
CFLAGS = ["-O2", "-std=c99", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]

OK = 0
BAD_ARG = 1
NONFINITE = 4


def build(source: str = SOURCE, output: str = LIBRARY, force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math, no FMA contraction)."""
    if not force and os.path.exists(output) and os.path.getmtime(output) >= os.path.getmtime(source):
        return output
    tmp = output + f".tmp{os.getpid()}"
    subprocess.run(["gcc", *CFLAGS, "-o", tmp, source, "-lm"], check=True)
    os.replace(tmp, output)
    return output


def build_variant(source_text: str) -> str:
    """Compile an edited copy of the oracle source into a temporary library
    (used by the tests that plant a mistake in the oracle)."""
    d = tempfile.mkdtemp(prefix="ttq_oracle_variant_")
    src = os.path.join(d, "variant.c")
    with open(src, "w") as f:
        f.write(source_text)
    return build(src, os.path.join(d, "libvariant.so"), force=True)


_P = ctypes.c_void_p
_I64 = ctypes.c_int64


class Oracle:
    """ctypes binding of one compiled oracle library."""

    def __init__(self, path: str | None = None):
        self.path = path or build()
        lib = ctypes.CDLL(self.path)
        lib.ttqo_f16_to_f32.argtypes = [ctypes.c_uint16]
        lib.ttqo_f16_to_f32.restype = ctypes.c_float
        lib.ttqo_f32_to_f16_ru.argtypes = [ctypes.c_float]
        lib.ttqo_f32_to_f16_ru.restype = ctypes.c_uint16
        lib.ttqo_act_norm.argtypes = [_P, _I64, _I64, ctypes.c_double, ctypes.c_double, ctypes.c_double, _P, _P]
        lib.ttqo_act_norm.restype = ctypes.c_int
        lib.ttqo_words_per_row.argtypes = [_I64, ctypes.c_int]
        lib.ttqo_words_per_row.restype = _I64
        lib.ttqo_code_at.argtypes = [_P, _I64, ctypes.c_int]
        lib.ttqo_code_at.restype = ctypes.c_int
        lib.ttqo_unpack.argtypes = [_P, _I64, _I64, ctypes.c_int, _P]
        lib.ttqo_unpack.restype = ctypes.c_int
        lib.ttqo_quantize.argtypes = [_P, _I64, _I64, _P, ctypes.c_int, ctypes.c_int, _P, _P, _P]
        lib.ttqo_quantize.restype = ctypes.c_int
        lib.ttqo_quantize_sym.argtypes = [_P, _I64, _I64, _P, ctypes.c_int, ctypes.c_int, _P, _P, _P]
        lib.ttqo_quantize_sym.restype = ctypes.c_int
        lib.ttqo_e4m3_value.argtypes = [ctypes.c_uint32]
        lib.ttqo_e4m3_value.restype = ctypes.c_double
        lib.ttqo_e4m3_from.argtypes = [ctypes.c_double]
        lib.ttqo_e4m3_from.restype = ctypes.c_uint32
        lib.ttqo_quantize_fp8.argtypes = [_P, _I64, _I64, _P, ctypes.c_int, _P, _P, _P]
        lib.ttqo_quantize_fp8.restype = ctypes.c_int
        lib.ttqo_dequant_rows_fp8.argtypes = [_P, _P, _P, _I64, _I64, ctypes.c_int, _P, _I64, _P]
        lib.ttqo_dequant_rows_fp8.restype = ctypes.c_int
        lib.ttqo_dequant_rows.argtypes = [_P, _P, _P, _P, _I64, _I64, ctypes.c_int, ctypes.c_int, _P, _I64, _P]
        lib.ttqo_dequant_rows.restype = ctypes.c_int
        lib.ttqo_project.argtypes = [_P, _I64, _P, _I64, _I64, _P]
        lib.ttqo_project.restype = ctypes.c_int
        lib.ttqo_lowrank_add.argtypes = [_P, _P, _I64, _I64, _P, _I64, _I64, _P]
        lib.ttqo_lowrank_add.restype = ctypes.c_int
        self.lib = lib

    # -- binary16 helpers ---------------------------------------------------
    def f16_to_f32(self, h: int) -> float:
        return float(self.lib.ttqo_f16_to_f32(int(h)))

    def f32_to_f16_ru(self, x: float) -> int:
        return int(self.lib.ttqo_f32_to_f16_ru(float(x)))

    def f16_array_to_f64(self, a: np.ndarray) -> np.ndarray:
        flat = np.ascontiguousarray(a, dtype=np.uint16).ravel()
        out = np.fromiter((self.lib.ttqo_f16_to_f32(int(v)) for v in flat), dtype=np.float64, count=flat.size)
        return out.reshape(np.shape(a))

    # -- method steps -------------------------------------------------------
    def act_norm(self, X: np.ndarray, p: float, lam: float, alpha: float):
        """D_ii = (||X_i,:||_p + lambda)^alpha and D^{-1/2}; X is [T][d]."""
        X = np.ascontiguousarray(X, dtype=np.float64)
        T, d = X.shape
        D = np.empty(d, np.float64)
        Dr = np.empty(d, np.float64)
        st = self.lib.ttqo_act_norm(X.ctypes.data, T, d, p, lam, alpha, D.ctypes.data, Dr.ctypes.data)
        return D, Dr, st

    def words_per_row(self, d: int, bits: int) -> int:
        return int(self.lib.ttqo_words_per_row(d, bits))

    def quantize(self, W: np.ndarray, D: np.ndarray | None, bits: int, group: int,
                 symmetric: bool = False):
        """Q[W D^{1/2}] in the binary32 operation order; W is [d'][d].
        symmetric=True: the symmetric quantiser (levels +-(2^(b-1)-1), zero
        point 2^(b-1) stored with the codes)."""
        W = np.ascontiguousarray(W, dtype=np.float32)
        dp, d = W.shape
        wpr = self.words_per_row(d, bits)
        codes = np.zeros((dp, wpr), np.uint32)
        ng = d // group if group > 0 and d % group == 0 else 1
        scales = np.zeros((dp, ng), np.uint16)
        zeros = np.zeros((dp, ng), np.uint16)
        Dp = None
        if D is not None:
            D32 = np.ascontiguousarray(D, dtype=np.float32)
            Dp = D32.ctypes.data
        fn = self.lib.ttqo_quantize_sym if symmetric else self.lib.ttqo_quantize
        st = fn(W.ctypes.data, dp, d, Dp, bits, group,
                codes.ctypes.data, scales.ctypes.data, zeros.ctypes.data)
        return codes, scales, zeros, st

    # -- FP8 (E4M3) codes --------------------------------------------------
    def e4m3_value(self, code: int) -> float:
        return float(self.lib.ttqo_e4m3_value(int(code)))

    def e4m3_from(self, v: float) -> int:
        return int(self.lib.ttqo_e4m3_from(float(v)))

    def quantize_fp8(self, W: np.ndarray, D: np.ndarray | None, group: int):
        """The E4M3 quantiser with the activation-aware scale; 8-bit codes
        packed 4 per word, zeros all binary16 +0."""
        W = np.ascontiguousarray(W, dtype=np.float32)
        dp, d = W.shape
        codes = np.zeros((dp, self.words_per_row(d, 8)), np.uint32)
        ng = d // group if group > 0 and d % group == 0 else 1
        scales = np.zeros((dp, ng), np.uint16)
        zeros = np.zeros((dp, ng), np.uint16)
        Dp = None
        if D is not None:
            D32 = np.ascontiguousarray(D, dtype=np.float32)
            Dp = D32.ctypes.data
        st = self.lib.ttqo_quantize_fp8(W.ctypes.data, dp, d, Dp, group, codes.ctypes.data,
                                        scales.ctypes.data, zeros.ctypes.data)
        return codes, scales, zeros, st

    def dequant_rows_fp8(self, codes, scales, Dr, d: int, group: int, rows=None):
        codes = np.ascontiguousarray(codes, dtype=np.uint32)
        scales = np.ascontiguousarray(scales, dtype=np.uint16)
        dp = codes.shape[0]
        rows_arr = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
        nrows = dp if rows is None else rows_arr.size
        What = np.empty((nrows, d), np.float64)
        Drp = None
        if Dr is not None:
            Dr64 = np.ascontiguousarray(Dr, dtype=np.float64)
            Drp = Dr64.ctypes.data
        st = self.lib.ttqo_dequant_rows_fp8(codes.ctypes.data, scales.ctypes.data, Drp, dp, d, group,
                                            None if rows_arr is None else rows_arr.ctypes.data, nrows,
                                            What.ctypes.data)
        if st != OK:
            raise ValueError(f"dequant_rows_fp8 failed ({st})")
        return What

    def code_at(self, codes_row: np.ndarray, i: int, bits: int) -> int:
        r = np.ascontiguousarray(codes_row, dtype=np.uint32)
        return int(self.lib.ttqo_code_at(r.ctypes.data, i, bits))

    def unpack(self, codes: np.ndarray, d: int, bits: int) -> np.ndarray:
        codes = np.ascontiguousarray(codes, dtype=np.uint32)
        out = np.empty((codes.shape[0], d), np.int32)
        st = self.lib.ttqo_unpack(codes.ctypes.data, codes.shape[0], d, bits, out.ctypes.data)
        if st != OK:
            raise ValueError(f"unpack failed ({st})")
        return out

    def dequant_rows(self, codes, scales, zeros, Dr, d: int, bits: int, group: int, rows=None):
        codes = np.ascontiguousarray(codes, dtype=np.uint32)
        scales = np.ascontiguousarray(scales, dtype=np.uint16)
        zeros = np.ascontiguousarray(zeros, dtype=np.uint16)
        dp = codes.shape[0]
        if rows is None:
            rows_arr = None
            nrows = dp
        else:
            rows_arr = np.ascontiguousarray(rows, dtype=np.int64)
            nrows = rows_arr.size
        What = np.empty((nrows, d), np.float64)
        Drp = None
        if Dr is not None:
            Dr64 = np.ascontiguousarray(Dr, dtype=np.float64)
            Drp = Dr64.ctypes.data
        st = self.lib.ttqo_dequant_rows(codes.ctypes.data, scales.ctypes.data, zeros.ctypes.data, Drp,
                                        dp, d, bits, group,
                                        None if rows_arr is None else rows_arr.ctypes.data, nrows,
                                        What.ctypes.data)
        if st != OK:
            raise ValueError(f"dequant_rows failed ({st})")
        return What

    def project(self, What: np.ndarray, X: np.ndarray) -> np.ndarray:
        What = np.ascontiguousarray(What, dtype=np.float64)
        X = np.ascontiguousarray(X, dtype=np.float64)
        nrows, d = What.shape
        T = X.shape[0]
        Y = np.empty((T, nrows), np.float64)
        st = self.lib.ttqo_project(What.ctypes.data, nrows, X.ctypes.data, T, d, Y.ctypes.data)
        if st != OK:
            raise ValueError(f"project failed ({st})")
        return Y

    def lowrank_add(self, A: np.ndarray, Brows: np.ndarray, X: np.ndarray, Y: np.ndarray) -> np.ndarray:
        A = np.ascontiguousarray(A, dtype=np.float64)
        Brows = np.ascontiguousarray(Brows, dtype=np.float64)
        X = np.ascontiguousarray(X, dtype=np.float64)
        Y = np.ascontiguousarray(Y, dtype=np.float64).copy()
        rank, d = A.shape
        T = X.shape[0]
        st = self.lib.ttqo_lowrank_add(A.ctypes.data, Brows.ctypes.data, rank, Brows.shape[0],
                                       X.ctypes.data, T, d, Y.ctypes.data)
        if st != OK:
            raise ValueError(f"lowrank_add failed ({st})")
        return Y

    # -- the whole layer ----------------------------------------------------
    def forward(self, X, W, p, lam, alpha, bits, group, A=None, B=None, rows=None,
                symmetric=False):
        """The TTQ linear layer for the listed output rows.

        Returns a dict with D, Dr (fp64), the codes/scales/zeros of all rows
        (the quantiser takes D rounded to binary32), and Y [T][len(rows)].
        """
        X = np.ascontiguousarray(X, dtype=np.float64)
        D, Dr, st1 = self.act_norm(X, p, lam, alpha)
        codes, scales, zeros, st2 = self.quantize(W, D.astype(np.float32), bits, group, symmetric)
        d = X.shape[1]
        What = self.dequant_rows(codes, scales, zeros, Dr, d, bits, group, rows)
        Y = self.project(What, X)
        if A is not None and B is not None and np.shape(A)[0] > 0:
            Bm = np.asarray(B, dtype=np.float64)
            Brows = Bm if rows is None else Bm[np.asarray(rows)]
            Y = self.lowrank_add(A, Brows, X, Y)
        return {"D": D, "Dr": Dr, "codes": codes, "scales": scales, "zeros": zeros,
                "Y": Y, "status": st1 | st2}


_default: Oracle | None = None


def get() -> Oracle:
    """The oracle built from this directory's source (compiled on first use)."""
    global _default
    if _default is None:
        _default = Oracle()
    return _default
