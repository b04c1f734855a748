"""Python binding of libttq.so: the C ABI of include/ttq.h, one function per
entry point with the same name.  Argument marshalling only -- every step of
the TTQ layer runs in the library's CUDA kernels; torch supplies device
memory and the current stream.  There is no fallback: if the library is
missing or the tensors are not on a CUDA device, the call raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIBRARY = os.path.join(_HERE, "libttq.so")

TTQ_OK = 0
TTQ_ERR_INVALID_ARG = 1
TTQ_ERR_UNSUPPORTED = 2
TTQ_ERR_CUDA = 3
TTQ_ERR_NONFINITE = 4
TTQ_ERR_TIMEOUT = 5
TTQ_ERR_WORKSPACE = 6

TTQ_F32 = 0
TTQ_BF16 = 1
TTQ_F16 = 2

TTQ_QSCHEME_ASYMMETRIC = 0
TTQ_QSCHEME_SYMMETRIC = 1
TTQ_QSCHEME_FP8_E4M3 = 2

TTQ_FLAG_NONFINITE = 0x1
TTQ_FLAG_SCALE_OVERFLOW = 0x2
TTQ_FLAG_TIMEOUT = 0x4
TTQ_FLAG_X_RANGE = 0x8
TTQ_FLAG_RANK_DEFICIENT = 0x10

# C signatures, in the order of include/ttq.h
_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_INT = ctypes.c_int
_F = ctypes.c_float
_SZ = ctypes.c_size_t


class WorkspaceLayout(ctypes.Structure):
    _fields_ = [("status", _SZ), ("D", _SZ), ("D_rsqrt", _SZ), ("partial", _SZ), ("codes", _SZ),
                ("scales", _SZ), ("zeros", _SZ), ("ax", _SZ), ("xh", _SZ), ("xb", _SZ), ("ab", _SZ),
                ("wq", _SZ), ("total", _SZ), ("splits", _I64), ("ax_ld", _I64), ("axp", _SZ),
                ("D_sqrt", _SZ), ("ypart", _SZ), ("tickets", _SZ), ("ax_splits", _I64)]


SIGNATURES = {
    "ttq_workspace_size": (_SZ, [_I64, _I64, _I64, _I64, _INT, _INT, _INT]),
    "ttq_workspace_get_layout": (_INT, [_I64, _I64, _I64, _I64, _INT, _INT, _INT,
                                        ctypes.POINTER(WorkspaceLayout)]),
    "ttq_workspace_init": (_INT, [_P, _SZ, _P]),
    "ttq_act_norm": (_INT, [_P, _INT, _I64, _I64, _F, _F, _F, _P, _P, _P, _SZ, _P]),
    "ttq_act_norm_noalloc": (_INT, [_P, _INT, _I64, _I64, _F, _F, _F, _P, _P, _P]),
    "ttq_act_norm_scale": (_INT, [_P, _INT, _I64, _I64, _F, _F, _F, _P, _P, _P, _P, _SZ, _P]),
    "ttq_quantize_weight": (_INT, [_P, _INT, _I64, _I64, _P, _INT, _INT, _P, _P, _P, _P, _SZ, _P]),
    "ttq_quantize_dequant_weight": (_INT, [_P, _INT, _I64, _I64, _P, _INT, _INT, _P, _P, _P, _P, _P,
                                           _SZ, _P]),
    "ttq_quantize_weight_ex": (_INT, [_P, _INT, _I64, _I64, _P, _INT, _INT, _INT, _P, _P, _P, _P, _P,
                                      _SZ, _P]),
    "ttq_linear_forward_ex": (_INT, [_P, _P, _P, _P, _INT, _I64, _I64, _I64, _I64, _F, _F, _F, _INT,
                                     _INT, _INT, _P, _INT, _P, _SZ, _P]),
    "ttq_dequantized_gemm": (_INT, [_P, _P, _I64, _I64, _I64, _P, _INT, _P, _SZ, _P]),
    "ttq_dequantized_gemm_workspace_size": (_SZ, [_I64, _I64, _I64]),
    "ttq_scale_activations": (_INT, [_P, _INT, _I64, _I64, _P, _P, _P, _SZ, _P]),
    "ttq_dequant_gemm": (_INT, [_P, _P, _P, _P, _P, _P, _P, _INT, _I64, _I64, _I64, _I64, _INT, _INT,
                                _P, _INT, _P, _SZ, _P]),
    "ttq_linear_forward": (_INT, [_P, _P, _P, _P, _INT, _I64, _I64, _I64, _I64, _F, _F, _F, _INT, _INT,
                                  _P, _INT, _P, _SZ, _P]),
    "ttq_linear_forward_kernels": (_INT, [_INT, _I64, _I64, _I64, _I64, _F, _INT, _INT, _INT,
                                          ctypes.POINTER(ctypes.c_int)]),
    "ttq_testing_wait_timeout": (_INT, [_INT, ctypes.c_uint64, _INT, _P, _SZ, _P]),
    "ttq_quantize_gemm": (_INT, [_P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _INT, _INT, _P, _P, _P,
                                 _P, _INT, _P, _SZ, _P]),
    "ttq_get_status": (_INT, [_P, ctypes.POINTER(ctypes.c_uint32)]),
    "ttq_status_from_flags": (_INT, [ctypes.c_uint32]),
    "ttq_lowrank_workspace_size": (_SZ, [_I64, _I64, _I64, _I64]),
    "ttq_lowrank_init": (_INT, [_P, _INT, _I64, _I64, _I64, _I64, _INT, _P, _P, _P, _P, _P, _SZ, _P]),
    "ttq_status_string": (ctypes.c_char_p, [_INT]),
    "ttq_version": (ctypes.c_char_p, []),
}

_lib = None


class TTQError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status) if _lib else status} ({status})")


def lib() -> ctypes.CDLL:
    """The loaded library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIBRARY):
            raise RuntimeError(f"libttq.so not found at {LIBRARY}; build it with "
                               "`python -m test_weight_quantization_ttq_b200.build`")
        L = ctypes.CDLL(LIBRARY)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def status_string(st: int) -> str:
    return lib().ttq_status_string(int(st)).decode()


def _check(st: int, where: str) -> None:
    if st != TTQ_OK:
        raise TTQError(st, where)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return TTQ_F32
    if t.dtype == torch.bfloat16:
        return TTQ_BF16
    if t.dtype == torch.float16:
        return TTQ_F16
    raise TypeError(f"unsupported dtype {t.dtype} (float32, bfloat16 or float16)")


def _dev(t: torch.Tensor | None, name: str) -> int | None:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    cur = torch.cuda.current_device()
    if t.device.index is not None and t.device.index != cur:
        raise ValueError(f"{name} is on {t.device}; the library runs on the current device cuda:{cur}")
    return t.data_ptr()


# The C ABI takes bare pointers and sizes, so the sizes it is given must
# describe the tensors behind the pointers: the checks below run before any
# device work and raise instead of letting a kernel read or write past a
# buffer.
_F32 = (torch.float32,)
_F16 = (torch.float16,)
_FLOAT_IN = (torch.float32, torch.bfloat16)


def _matrix(t: torch.Tensor | None, name: str, rows=None, cols=None, dtypes=None) -> None:
    """t (when given) is 2-D, rows x cols where those are given, of one of `dtypes`."""
    if t is None:
        return
    if t.dim() != 2:
        raise ValueError(f"{name} must be 2-D, got shape {tuple(t.shape)}")
    if (rows is not None and t.shape[0] != rows) or (cols is not None and t.shape[1] != cols):
        want = (rows if rows is not None else "*", cols if cols is not None else "*")
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {want}")
    if dtypes is not None and t.dtype not in dtypes:
        raise TypeError(f"{name} has dtype {t.dtype}, expected one of {list(dtypes)}")


def _vector(t: torch.Tensor | None, name: str, n: int) -> None:
    """t (when given) holds exactly n float32 values (D, D^{-1/2})."""
    if t is None:
        return
    if t.dtype != torch.float32 or t.numel() != n:
        raise ValueError(f"{name} must hold {n} float32 values, got {t.numel()} {t.dtype}")


def _room(t: torch.Tensor | None, name: str, nbytes: int) -> None:
    """t (when given) spans at least nbytes (packed codes, binary16 scales)."""
    if t is None:
        return
    if t.numel() * t.element_size() < nbytes:
        raise ValueError(f"{name} spans {t.numel() * t.element_size()} bytes, needs {nbytes}")


def _qsizes(d: int, bits: int, group: int, where: str) -> tuple[int, int]:
    """(code bytes, scale bytes) of one row of W."""
    if bits < 1 or group < 1:
        raise TTQError(TTQ_ERR_INVALID_ARG, where)
    return d * bits // 32 * 4, d // group * 2


def _lowrank_pair(A: torch.Tensor | None, B: torch.Tensor | None) -> int:
    """r of the low-rank term: A [r][d] and B [d'][r] are given together."""
    if (A is None) != (B is None):
        raise ValueError("A and B of the low-rank term are given together or not at all")
    return 0 if A is None else A.shape[0]


def _nbytes(ws: torch.Tensor) -> int:
    return ws.numel() * ws.element_size()


def _stream(stream) -> int | None:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream or None


# ------------------------------------------------------------- workspace
def ttq_workspace_size(d, dp, T, r, bits, group, dtype=TTQ_BF16) -> int:
    return int(lib().ttq_workspace_size(d, dp, T, r, bits, group, dtype))


def ttq_workspace_get_layout(d, dp, T, r, bits, group, dtype=TTQ_BF16) -> WorkspaceLayout:
    out = WorkspaceLayout()
    _check(lib().ttq_workspace_get_layout(d, dp, T, r, bits, group, dtype, ctypes.byref(out)),
           "ttq_workspace_get_layout")
    return out


def ttq_workspace_init(ws: torch.Tensor, stream=None) -> None:
    _check(lib().ttq_workspace_init(_dev(ws, "ws"), _nbytes(ws), _stream(stream)), "ttq_workspace_init")


def new_workspace(d, dp, T, r, bits, group, dtype=TTQ_BF16, device="cuda", stream=None) -> torch.Tensor:
    """A zero-initialised workspace (uint8 tensor) for this shape."""
    n = ttq_workspace_size(d, dp, T, r, bits, group, dtype)
    if n == 0:
        raise TTQError(TTQ_ERR_INVALID_ARG, "ttq_workspace_size")
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    ttq_workspace_init(ws, stream)
    return ws


def ttq_get_status(ws: torch.Tensor) -> tuple[int, int]:
    """(status, raw flag bits) of the workspace; synchronise the stream first."""
    flags = ctypes.c_uint32(0)
    st = lib().ttq_get_status(_dev(ws, "ws"), ctypes.byref(flags))
    return int(st), int(flags.value)


def ttq_status_from_flags(flags: int) -> int:
    """The status a set of TTQ_FLAG_* bits stands for (host only)."""
    return int(lib().ttq_status_from_flags(int(flags) & 0xFFFFFFFF))


# ---------------------------------------------------------- entry points
def _quant_outputs(dp, d, D, bits, group, codes, scales, zeros, W_hat, where) -> None:
    cb, sb = _qsizes(d, bits, group, where)
    _vector(D, "D", d)
    _room(codes, "codes", dp * cb)
    _room(scales, "scales", dp * sb)
    _room(zeros, "zeros", dp * sb)
    _matrix(W_hat, "W_hat", dp, d, _F16)


def ttq_act_norm(X, p, lam, alpha, ws=None, D=None, D_rsqrt=None, stream=None, copy_out=True):
    """D[i] = (||X[:, i]||_p + lambda)^alpha and D^{-1/2}; X is [T][d].
    With copy_out=False nothing is copied out: D and D^{-1/2} are returned
    as views of the workspace, where the entry point writes them."""
    _matrix(X, "X", dtypes=_FLOAT_IN)
    T, d = X.shape
    _vector(D, "D", d)
    _vector(D_rsqrt, "D_rsqrt", d)
    if ws is None:
        ws = new_workspace(d, 0, T, 0, 4, 32, _dtype_code(X), X.device, stream)
    if not copy_out:
        _check(lib().ttq_act_norm(_dev(X, "X"), _dtype_code(X), d, T, p, lam, alpha, None, None,
                                  _dev(ws, "ws"), _nbytes(ws), _stream(stream)), "ttq_act_norm")
        L = ttq_workspace_get_layout(d, 0, T, 0, 4, 32, _dtype_code(X))
        return (ws[L.D: L.D + 4 * d].view(torch.float32), ws[L.D_rsqrt: L.D_rsqrt + 4 * d].view(torch.float32))
    if D is None:
        D = torch.empty(d, dtype=torch.float32, device=X.device)
    if D_rsqrt is None:
        D_rsqrt = torch.empty(d, dtype=torch.float32, device=X.device)
    _check(lib().ttq_act_norm(_dev(X, "X"), _dtype_code(X), d, T, p, lam, alpha, _dev(D, "D"),
                              _dev(D_rsqrt, "D_rsqrt"), _dev(ws, "ws"), _nbytes(ws), _stream(stream)),
           "ttq_act_norm")
    return D, D_rsqrt


def ttq_act_norm_scale(X, p, lam, alpha, ws=None, D=None, D_rsqrt=None, Xs=None, stream=None,
                       copy_out=True):
    """D, D^{-1/2} and Xs [T][d] binary16 = X * D^{-1/2} in one pass over X.
    With copy_out=False, D and D^{-1/2} are not given to the entry point and
    are returned as views of the workspace, where it writes them."""
    _matrix(X, "X", dtypes=_FLOAT_IN)
    T, d = X.shape
    _vector(D, "D", d)
    _vector(D_rsqrt, "D_rsqrt", d)
    _matrix(Xs, "Xs", T, d, _F16)
    if ws is None:
        ws = new_workspace(d, 0, T, 0, 4, 32, _dtype_code(X), X.device, stream)
    if Xs is None:
        Xs = torch.empty((T, d), dtype=torch.float16, device=X.device)
    if copy_out:
        if D is None:
            D = torch.empty(d, dtype=torch.float32, device=X.device)
        if D_rsqrt is None:
            D_rsqrt = torch.empty(d, dtype=torch.float32, device=X.device)
        dptr, drptr = _dev(D, "D"), _dev(D_rsqrt, "D_rsqrt")
    else:
        dptr = drptr = None
    _check(lib().ttq_act_norm_scale(_dev(X, "X"), _dtype_code(X), d, T, p, lam, alpha, dptr, drptr,
                                    _dev(Xs, "Xs"), _dev(ws, "ws"), _nbytes(ws), _stream(stream)),
           "ttq_act_norm_scale")
    if not copy_out:
        L = ttq_workspace_get_layout(d, 0, T, 0, 4, 32, _dtype_code(X))
        D = ws[L.D: L.D + 4 * d].view(torch.float32)
        D_rsqrt = ws[L.D_rsqrt: L.D_rsqrt + 4 * d].view(torch.float32)
    return D, D_rsqrt, Xs


def ttq_linear_forward_kernels(d, dp, T, r=0, p=2.0, dtype=TTQ_BF16, bits=4, group=128,
                               scheme=TTQ_QSCHEME_ASYMMETRIC) -> int:
    """Kernels one ttq_linear_forward(_ex) call of these sizes and this code
    scheme enqueues on the current device."""
    n = ctypes.c_int(0)
    _check(lib().ttq_linear_forward_kernels(dtype, d, dp, T, r, p, bits, group, scheme, ctypes.byref(n)),
           "ttq_linear_forward_kernels")
    return n.value


def ttq_act_norm_noalloc(X, p, lam, alpha, D=None, D_rsqrt=None, stream=None):
    """ttq_act_norm without a workspace: the library's own fixed scratch array
    is used (d <= 16384; calls overlapping on the GPU race)."""
    _matrix(X, "X", dtypes=_FLOAT_IN)
    T, d = X.shape
    _vector(D, "D", d)
    _vector(D_rsqrt, "D_rsqrt", d)
    if D is None:
        D = torch.empty(d, dtype=torch.float32, device=X.device)
    if D_rsqrt is None:
        D_rsqrt = torch.empty(d, dtype=torch.float32, device=X.device)
    _check(lib().ttq_act_norm_noalloc(_dev(X, "X"), _dtype_code(X), d, T, p, lam, alpha, _dev(D, "D"),
                                      _dev(D_rsqrt, "D_rsqrt"), _stream(stream)),
           "ttq_act_norm_noalloc")
    return D, D_rsqrt


def ttq_quantize_weight(W, D, bits, group, ws=None, codes=None, scales=None, zeros=None, stream=None):
    """codes [d'][d*bits/32] uint32, scales/zeros [d'][d/group] binary16 bits (int16 storage)."""
    _matrix(W, "W", dtypes=_FLOAT_IN)
    dp, d = W.shape
    _quant_outputs(dp, d, D, bits, group, codes, scales, zeros, None, "ttq_quantize_weight")
    dev = W.device
    if ws is None:
        ws = new_workspace(d, 0, 0, 0, bits, group, _dtype_code(W), dev, stream)
    if codes is None:
        codes = torch.empty((dp, d * bits // 32), dtype=torch.int32, device=dev)
    if scales is None:
        scales = torch.empty((dp, d // group), dtype=torch.int16, device=dev)
    if zeros is None:
        zeros = torch.empty((dp, d // group), dtype=torch.int16, device=dev)
    _check(lib().ttq_quantize_weight(_dev(W, "W"), _dtype_code(W), dp, d, _dev(D, "D"), bits, group,
                                     _dev(codes, "codes"), _dev(scales, "scales"), _dev(zeros, "zeros"),
                                     _dev(ws, "ws"), _nbytes(ws), _stream(stream)),
           "ttq_quantize_weight")
    return codes, scales, zeros


def ttq_quantize_weight_ex(W, D, bits, group, scheme, ws=None, codes=None, scales=None, zeros=None,
                           W_hat=None, stream=None, with_codes=True):
    """Codes, scales and zeros under the given TTQ_QSCHEME_*; W_hat (binary16
    s (q - z), optional) is written when given.  With with_codes=False (and
    W_hat given) only W_hat is written and (None, None, None) is returned."""
    _matrix(W, "W", dtypes=_FLOAT_IN)
    dp, d = W.shape
    _quant_outputs(dp, d, D, bits, group, codes, scales, zeros, W_hat, "ttq_quantize_weight_ex")
    dev = W.device
    if ws is None:
        ws = new_workspace(d, 0, 0, 0, bits, group, _dtype_code(W), dev, stream)
    if not with_codes:
        if W_hat is None:
            raise ValueError("ttq_quantize_weight_ex: with_codes=False needs W_hat")
        _check(lib().ttq_quantize_weight_ex(
            _dev(W, "W"), _dtype_code(W), dp, d, _dev(D, "D"), bits, group, scheme, None, None, None,
            _dev(W_hat, "W_hat"), _dev(ws, "ws"), _nbytes(ws), _stream(stream)), "ttq_quantize_weight_ex")
        return None, None, None
    if codes is None:
        codes = torch.empty((dp, d * bits // 32), dtype=torch.int32, device=dev)
    if scales is None:
        scales = torch.empty((dp, d // group), dtype=torch.int16, device=dev)
    if zeros is None:
        zeros = torch.empty((dp, d // group), dtype=torch.int16, device=dev)
    _check(lib().ttq_quantize_weight_ex(
        _dev(W, "W"), _dtype_code(W), dp, d, _dev(D, "D"), bits, group, scheme, _dev(codes, "codes"),
        _dev(scales, "scales"), _dev(zeros, "zeros"), _dev(W_hat, "W_hat"), _dev(ws, "ws"), _nbytes(ws),
        _stream(stream)), "ttq_quantize_weight_ex")
    return codes, scales, zeros


def ttq_quantize_dequant_weight(W, D, bits, group, ws=None, codes=None, scales=None, zeros=None,
                                W_hat=None, stream=None, with_codes=True):
    """ttq_quantize_weight plus W_hat [d'][d] binary16 (torch.float16) = s (q - z).
    With with_codes=False only W_hat is written (codes, scales, zeros are None)."""
    _matrix(W, "W", dtypes=_FLOAT_IN)
    dp, d = W.shape
    _quant_outputs(dp, d, D, bits, group, codes, scales, zeros, W_hat, "ttq_quantize_dequant_weight")
    dev = W.device
    if ws is None:
        ws = new_workspace(d, 0, 0, 0, bits, group, _dtype_code(W), dev, stream)
    if W_hat is None:
        W_hat = torch.empty((dp, d), dtype=torch.float16, device=dev)
    if not with_codes:
        _check(lib().ttq_quantize_dequant_weight(
            _dev(W, "W"), _dtype_code(W), dp, d, _dev(D, "D"), bits, group, None, None, None,
            _dev(W_hat, "W_hat"), _dev(ws, "ws"), _nbytes(ws), _stream(stream)),
            "ttq_quantize_dequant_weight")
        return None, None, None, W_hat
    if codes is None:
        codes = torch.empty((dp, d * bits // 32), dtype=torch.int32, device=dev)
    if scales is None:
        scales = torch.empty((dp, d // group), dtype=torch.int16, device=dev)
    if zeros is None:
        zeros = torch.empty((dp, d // group), dtype=torch.int16, device=dev)
    if W_hat is None:
        W_hat = torch.empty((dp, d), dtype=torch.float16, device=dev)
    _check(lib().ttq_quantize_dequant_weight(
        _dev(W, "W"), _dtype_code(W), dp, d, _dev(D, "D"), bits, group, _dev(codes, "codes"),
        _dev(scales, "scales"), _dev(zeros, "zeros"), _dev(W_hat, "W_hat"), _dev(ws, "ws"),
        _nbytes(ws), _stream(stream)), "ttq_quantize_dequant_weight")
    return codes, scales, zeros, W_hat


def ttq_dequantized_gemm(W_hat, Xs, ws=None, Y=None, y_dtype=torch.bfloat16, stream=None):
    """Y [T][d'] = W_hat Xs^T from a binary16 dequantised weight and binary16 X D^{-1/2}."""
    _matrix(W_hat, "W_hat", dtypes=_F16)
    dp, d = W_hat.shape
    _matrix(Xs, "Xs", cols=d, dtypes=_F16)
    T = Xs.shape[0]
    _matrix(Y, "Y", T, dp, _FLOAT_IN)
    if ws is None:
        # room for the forward's K split of this shape, so the result is its bits
        nbytes = max(4096, int(lib().ttq_dequantized_gemm_workspace_size(d, dp, T)))
        ws = torch.empty(nbytes, dtype=torch.uint8, device=W_hat.device)
        ttq_workspace_init(ws, stream)
    if Y is None:
        Y = torch.empty((T, dp), dtype=y_dtype, device=W_hat.device)
    _check(lib().ttq_dequantized_gemm(_dev(W_hat, "W_hat"), _dev(Xs, "Xs"), d, dp, T, _dev(Y, "Y"),
                                      _dtype_code(Y), _dev(ws, "ws"), _nbytes(ws), _stream(stream)),
           "ttq_dequantized_gemm")
    return Y


def ttq_scale_activations(X, D_rsqrt, ws=None, Xs=None, stream=None):
    """Xs [T][d] binary16 (torch.float16) = X * D^{-1/2}, the product's B operand."""
    _matrix(X, "X", dtypes=_FLOAT_IN + _F16)
    T, d = X.shape
    _vector(D_rsqrt, "D_rsqrt", d)
    _matrix(Xs, "Xs", T, d, _F16)
    if ws is None:
        ws = new_workspace(d, 0, 0, 0, 4, 32, TTQ_BF16, X.device, stream)
    if Xs is None:
        Xs = torch.empty((T, d), dtype=torch.float16, device=X.device)
    _check(lib().ttq_scale_activations(_dev(X, "X"), _dtype_code(X), d, T, _dev(D_rsqrt, "D_rsqrt"),
                                       _dev(Xs, "Xs"), _dev(ws, "ws"), _nbytes(ws), _stream(stream)),
           "ttq_scale_activations")
    return Xs


def ttq_dequant_gemm(codes, scales, zeros, D_rsqrt, X, A, B, bits, group, ws=None, Y=None,
                     y_dtype=None, stream=None):
    """Y [T][d'] = W_hat X (+ B (A X)) from quantised weights; Y in y_dtype
    (default: the dtype of X, or of a given Y)."""
    _matrix(X, "X", dtypes=_FLOAT_IN + _F16)
    T, d = X.shape
    dp = codes.shape[0]
    r = _lowrank_pair(A, B)
    cb, sb = _qsizes(d, bits, group, "ttq_dequant_gemm")
    _room(codes, "codes", dp * cb)
    _room(scales, "scales", dp * sb)
    _room(zeros, "zeros", dp * sb)
    _vector(D_rsqrt, "D_rsqrt", d)
    _matrix(A, "A", r, d, (X.dtype,))
    _matrix(B, "B", dp, r, (X.dtype,))
    _matrix(Y, "Y", T, dp, _FLOAT_IN)
    dt = _dtype_code(X)
    if ws is None:
        ws = new_workspace(d, dp, T, r, bits, group, dt, X.device, stream)
    if Y is None:
        Y = torch.empty((T, dp), dtype=y_dtype or (torch.bfloat16 if dt == TTQ_F16 else X.dtype),
                        device=X.device)
    _check(lib().ttq_dequant_gemm(_dev(codes, "codes"), _dev(scales, "scales"), _dev(zeros, "zeros"),
                                  _dev(D_rsqrt, "D_rsqrt"), _dev(X, "X"), _dev(A, "A"), _dev(B, "B"), dt,
                                  d, dp, T, r, bits, group, _dev(Y, "Y"), _dtype_code(Y), _dev(ws, "ws"),
                                  _nbytes(ws), _stream(stream)),
           "ttq_dequant_gemm")
    return Y


TTQ_TESTING_WAIT_MBARRIER = 0


def ttq_testing_wait_timeout(kind, limit_ns, blocks, ws, stream=None) -> None:
    """Test hook: `blocks` blocks each make one wait of `kind` that cannot
    complete, with a limit of limit_ns; they set TTQ_FLAG_TIMEOUT in ws."""
    _check(lib().ttq_testing_wait_timeout(kind, limit_ns, blocks, _dev(ws, "ws"), _nbytes(ws),
                                          _stream(stream)), "ttq_testing_wait_timeout")


def ttq_quantize_gemm(W, D, Xs, A, B, X, bits, group, ws=None, Y=None, y_dtype=torch.bfloat16,
                      codes=None, scales=None, zeros=None, stream=None):
    """Steps (2)-(3) in one pass over bf16 W [d'][d] for T <= 16 tokens:
    Y [T][d'] = Q[W D^{1/2}] Xs (+ B (A X)), Xs the binary16 X D^{-1/2}
    [T][d]; A [r][d], B [d'][r], X [T][d] bf16 for the low-rank term.
    codes/scales/zeros: None, or all three buffers to receive the codes."""
    _matrix(Xs, "Xs", dtypes=_F16)
    T, d = Xs.shape
    _matrix(W, "W", cols=d, dtypes=(torch.bfloat16,))
    dp = W.shape[0]
    _vector(D, "D", d)
    r = _lowrank_pair(A, B)
    _matrix(A, "A", r, d, (torch.bfloat16,))
    _matrix(B, "B", dp, r, (torch.bfloat16,))
    if r > 0:
        _matrix(X, "X", T, d, (torch.bfloat16,))
    given = [t is not None for t in (codes, scales, zeros)]
    if any(given) and not all(given):
        raise TTQError(TTQ_ERR_INVALID_ARG, "ttq_quantize_gemm: codes, scales and zeros go together")
    if all(given):
        cb, sb = _qsizes(d, bits, group, "ttq_quantize_gemm")
        _room(codes, "codes", dp * cb)
        _room(scales, "scales", dp * sb)
        _room(zeros, "zeros", dp * sb)
    _matrix(Y, "Y", T, dp, _FLOAT_IN)
    if ws is None:
        ws = new_workspace(d, dp, T, r, bits, group, TTQ_BF16, W.device, stream)
    if Y is None:
        Y = torch.empty((T, dp), dtype=y_dtype, device=W.device)
    _check(lib().ttq_quantize_gemm(_dev(W, "W"), _dev(D, "D"), _dev(Xs, "Xs"), _dev(A, "A"), _dev(B, "B"),
                                   _dev(X if r > 0 else None, "X"), d, dp, T, r, bits, group,
                                   _dev(codes, "codes"), _dev(scales, "scales"), _dev(zeros, "zeros"),
                                   _dev(Y, "Y"), _dtype_code(Y), _dev(ws, "ws"), _nbytes(ws),
                                   _stream(stream)),
           "ttq_quantize_gemm")
    return Y


def ttq_linear_forward(X, W, A, B, p, lam, alpha, bits, group, ws=None, Y=None, y_dtype=None,
                       stream=None, scheme=None):
    """The TTQ linear layer: Y [T][d'] = Q[W D^{1/2}] D^{-1/2} X + B (A X);
    Y in y_dtype (default: the dtype of X, or of a given Y).  scheme: None
    (ttq_linear_forward) or a TTQ_QSCHEME_* code (ttq_linear_forward_ex)."""
    _matrix(X, "X", dtypes=_FLOAT_IN)
    T, d = X.shape
    _matrix(W, "W", cols=d, dtypes=(X.dtype,))
    dp = W.shape[0]
    r = _lowrank_pair(A, B)
    _matrix(A, "A", r, d, (X.dtype,))
    _matrix(B, "B", dp, r, (X.dtype,))
    _matrix(Y, "Y", T, dp, _FLOAT_IN)
    dt = _dtype_code(X)
    if ws is None:
        ws = new_workspace(d, dp, T, r, bits, group, dt, X.device, stream)
    if Y is None:
        Y = torch.empty((T, dp), dtype=y_dtype or X.dtype, device=X.device)
    args = (_dev(X, "X"), _dev(W, "W"), _dev(A, "A"), _dev(B, "B"), dt, d, dp, T, r, p, lam, alpha, bits,
            group)
    tail = (_dev(Y, "Y"), _dtype_code(Y), _dev(ws, "ws"), _nbytes(ws), _stream(stream))
    if scheme is None:
        _check(lib().ttq_linear_forward(*args, *tail), "ttq_linear_forward")
    else:
        _check(lib().ttq_linear_forward_ex(*args, scheme, *tail), "ttq_linear_forward_ex")
    return Y


def ttq_lowrank_workspace_size(dp, d, r, oversample) -> int:
    return int(lib().ttq_lowrank_workspace_size(dp, d, r, oversample))


def ttq_lowrank_init(W, r, Omega, power_iters=2, ws=None, B=None, A=None, W_res=None,
                     residual=True, stream=None):
    """Static low-rank factors of W [d'][d] (float32 or bf16): B [d'][r],
    A [r][d] from a randomised truncated SVD with the Gaussian test matrix
    Omega [d][r + oversample] (float32), and W_res = W - B A (when
    `residual`).  Returns (B, A, W_res or None)."""
    _matrix(W, "W", dtypes=_FLOAT_IN)
    dp, d = W.shape
    _matrix(Omega, "Omega", d, None, _F32)
    _matrix(B, "B", dp, r, (W.dtype,))
    _matrix(A, "A", r, d, (W.dtype,))
    _matrix(W_res, "W_res", dp, d, (W.dtype,))
    l = Omega.shape[1]
    oversample = l - r
    dt = _dtype_code(W)
    if ws is None:
        n = ttq_lowrank_workspace_size(dp, d, r, oversample)
        if n == 0:
            raise TTQError(TTQ_ERR_INVALID_ARG, "ttq_lowrank_workspace_size")
        ws = torch.empty(n, dtype=torch.uint8, device=W.device)
        ttq_workspace_init(ws, stream)
    if B is None:
        B = torch.empty((dp, r), dtype=W.dtype, device=W.device)
    if A is None:
        A = torch.empty((r, d), dtype=W.dtype, device=W.device)
    if W_res is None and residual:
        W_res = torch.empty_like(W)
    _check(lib().ttq_lowrank_init(_dev(W, "W"), dt, dp, d, r, oversample, power_iters, _dev(Omega, "Omega"),
                                  _dev(B, "B"), _dev(A, "A"), _dev(W_res, "W_res"), _dev(ws, "ws"),
                                  _nbytes(ws), _stream(stream)),
           "ttq_lowrank_init")
    return B, A, W_res


def workspace_views(ws: torch.Tensor, d, dp, T, r, bits, group, dtype=TTQ_BF16) -> dict:
    """Views of the intermediates a forward call leaves in its workspace."""
    L = ttq_workspace_get_layout(d, dp, T, r, bits, group, dtype)

    def view(off, n, dt):
        itemsize = torch.empty((), dtype=dt).element_size()
        return ws[off: off + n * itemsize].view(dt)

    out = {"D": view(L.D, d, torch.float32), "D_rsqrt": view(L.D_rsqrt, d, torch.float32)}
    if dp > 0:
        out["codes"] = view(L.codes, dp * (d * bits // 32), torch.int32).view(dp, -1)
        out["scales"] = view(L.scales, dp * (d // group), torch.int16).view(dp, -1)
        out["zeros"] = view(L.zeros, dp * (d // group), torch.int16).view(dp, -1)
        out["xh"] = view(L.xh, T * d, torch.float16).view(T, d)
        if L.wq:
            out["wq"] = view(L.wq, dp * d, torch.float16).view(dp, d)
    return out
