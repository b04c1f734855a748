"""The C ABI library on the CPU: it loads, exports every entry point that
include/*.h declare, and its host-side logic (workspace layout, argument
checks that reject before any device work) behaves as documented.  No
compute call is made here."""
import os
import re

import pytest

from test_weight_quantization_ttq_b200 import build as ttq_build
from test_weight_quantization_ttq_b200 import ttq

INCLUDE = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")
HEADERS = sorted(os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE) if f.endswith(".h"))


def _header_text():
    return "".join(open(h).read() for h in HEADERS)


@pytest.fixture(scope="module")
def L():
    ttq_build.build()
    return ttq.lib()


def declared_functions():
    text = _header_text()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ttq_[a-z_0-9]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert len(names) >= 9, names
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(ttq.SIGNATURES), "binding and header disagree"


def test_version_and_status_strings(L):
    assert ttq.lib().ttq_version().decode().count(".") == 2
    for st in range(7):
        assert ttq.status_string(st)
    assert ttq.status_string(99) == "unknown status"


def test_status_from_flags(L):
    f = ttq.ttq_status_from_flags
    assert f(0) == ttq.TTQ_OK
    # a weight of low rank is a warning, not an error
    assert f(ttq.TTQ_FLAG_RANK_DEFICIENT) == ttq.TTQ_OK
    for bit in (ttq.TTQ_FLAG_NONFINITE, ttq.TTQ_FLAG_SCALE_OVERFLOW, ttq.TTQ_FLAG_X_RANGE, 0x80000000):
        assert f(bit) == ttq.TTQ_ERR_NONFINITE, bit
        assert f(bit | ttq.TTQ_FLAG_RANK_DEFICIENT) == ttq.TTQ_ERR_NONFINITE, bit
    # a timed-out wait outranks every other condition
    assert f(ttq.TTQ_FLAG_TIMEOUT | ttq.TTQ_FLAG_NONFINITE | ttq.TTQ_FLAG_RANK_DEFICIENT) == ttq.TTQ_ERR_TIMEOUT


def test_workspace_layout_is_consistent(L):
    for (d, dp, T, r, bits, g, dt) in [(4096, 4096, 2048, 0, 4, 128, ttq.TTQ_BF16),
                                       (8192, 28672, 4096, 64, 2, 64, ttq.TTQ_BF16),
                                       (256, 256, 64, 0, 4, 64, ttq.TTQ_F32),
                                       (96, 200, 0, 8, 3, 32, ttq.TTQ_F32)]:
        n = ttq.ttq_workspace_size(d, dp, T, r, bits, g, dt)
        lay = ttq.ttq_workspace_get_layout(d, dp, T, r, bits, g, dt)
        assert n == lay.total > 0
        offs = [lay.status, lay.D, lay.D_rsqrt, lay.partial, lay.codes, lay.scales, lay.zeros]
        assert all(o % 256 == 0 for o in offs)
        assert offs == sorted(offs) and len(set(offs)) == len(offs)
        assert lay.codes + dp * d * bits // 8 <= lay.scales
        assert lay.scales + dp * (d // g) * 2 <= lay.zeros
        assert lay.partial + 8 * lay.splits * d <= lay.codes
        if r:
            assert lay.ax_ld == r and lay.ax >= lay.zeros + dp * (d // g) * 2
        if T and dp:
            assert lay.xh > 0
        if dt == ttq.TTQ_F32 and r:
            assert lay.xb > 0 and lay.ab > 0


@pytest.mark.parametrize("d,T,splits", [
    (4096, 2048, 8),     # 32 column blocks of 128 channels: 8 splits of 256 rows (one cluster)
    (8192, 2048, 8),     # 256 rows per split still needs 8 splits
    (4096, 1024, 8),     # two blocks per SM would take 10: capped at a cluster of 8
    (4096, 150, 5),      # no more splits than ceil(T / 32): 5 of 30 rows
    (4096, 16, 1),
    (4096, 0, 1),
    (4096, 4096, 16),    # too many rows for 8 splits of 256: 16 blocks of 256 channels x 16
    (8192, 8192, 9),     # 32 blocks of 256 channels: 9 splits keep 288 blocks in one wave
    (11008, 512, 3),     # 86 blocks of 128 channels: 3 splits keep 258 blocks in one wave
])
def test_statistic_split_plan(L, d, T, splits):
    """The token splits of the statistic pass: the fused kernel's clusters
    hold at most 8 splits of at most 256 rows, and the blocks fit two per SM
    in one wave where the rows allow."""
    lay = ttq.ttq_workspace_get_layout(d, 0, T, 0, 4, 32, ttq.TTQ_BF16)
    assert lay.splits == splits
    if T:
        rps = -(-T // splits)
        assert -(-T // rps) == splits and splits <= -(-T // 32)


def test_dequantised_weight_only_for_long_inputs(L):
    """The forward materialises s (q - z) only for more than 256 tokens."""
    for T in (0, 1, 16, 256):
        assert ttq.ttq_workspace_get_layout(4096, 4096, T, 0, 4, 128, ttq.TTQ_BF16).wq == 0
    lay = ttq.ttq_workspace_get_layout(4096, 4096, 257, 0, 4, 128, ttq.TTQ_BF16)
    assert lay.wq % 256 == 0 and lay.wq > lay.zeros and lay.wq + 4096 * 4096 * 2 <= lay.total


def test_split_product_plan(L):
    """The product on the materialised weight splits along K where few output
    rows meet a long K, and only there: the 11008 -> 4096 projection at 512
    tokens in 4 splits (its float32 partial sums in the layout's ypart
    region, 4 x 512 x 4096 floats, and the same room after the 20 KiB header
    for ttq_dequantized_gemm), the 4096 -> 4096 and 4096 -> 11008 layers and
    the 8192 -> 28672 ones not at all."""
    lay = ttq.ttq_workspace_get_layout(11008, 4096, 512, 32, 3, 128, ttq.TTQ_BF16)
    need = 4 * 512 * 4096 * 4
    assert lay.ypart % 256 == 0 and lay.ypart > lay.wq and lay.ypart + need <= lay.total
    assert L.ttq_dequantized_gemm_workspace_size(11008, 4096, 512) == 20480 + need
    for d, dp, T, r in ((4096, 4096, 2048, 0), (4096, 11008, 512, 32), (8192, 28672, 1024, 64),
                        (8192, 28672, 4096, 64)):
        assert ttq.ttq_workspace_get_layout(d, dp, T, r, 3, 128, ttq.TTQ_BF16).ypart == 0, (d, dp, T)
        assert L.ttq_dequantized_gemm_workspace_size(d, dp, T) == 4096, (d, dp, T)
    # at most 256 tokens the product is never split
    assert ttq.ttq_workspace_get_layout(11008, 4096, 256, 32, 3, 128, ttq.TTQ_BF16).ypart == 0
    assert L.ttq_dequantized_gemm_workspace_size(11008, 4096, 256) == 4096
    assert L.ttq_dequantized_gemm_workspace_size(12, 4096, 512) == 0   # d % 8 != 0


def test_low_rank_product_parts(L):
    """A X's reduction over d: for 17 to 512 tokens the warp-level MMA
    kernel's channel slices (512 channels for r <= 32, 256 above), whose
    partial sums the layout holds; otherwise the tensor-core GEMM's K splits
    (at most one wave, at least 4 blocks of 64 channels each)."""
    def lay(d, T, r):
        return ttq.ttq_workspace_get_layout(d, 4096, T, r, 3, 128, ttq.TTQ_BF16)
    for d, T, r, parts in ((4096, 512, 32, 8), (11008, 512, 32, 22), (8192, 128, 64, 32),
                           (448 + 64, 77, 16, 1), (4096, 17, 96, 16)):
        lo = lay(d, T, r)
        assert lo.ax_splits == parts, (d, T, r, lo.ax_splits)
        if parts > 1:
            assert lo.axp % 256 == 0 and lo.axp + parts * T * r * 4 <= lo.total
        else:
            assert lo.axp == 0
    for d, T, r in ((8192, 1, 64), (8192, 16, 64), (4096, 513, 32), (8192, 4096, 64)):
        lo = lay(d, T, r)
        kb = -(-d // 64)
        assert 1 <= lo.ax_splits <= max(1, kb // 4), (d, T, r, lo.ax_splits)


@pytest.mark.parametrize("args", [
    (4096, 4096, 2048, 0, 5, 128),   # bits not built
    (4096, 4096, 2048, 0, 4, 96),    # group not built
    (4100, 4096, 2048, 0, 4, 128),   # d % group
    (4096, 4096, 2048, 4, 4, 128),   # rank not a multiple of 8
    (4096, -1, 2048, 0, 4, 128),
])
def test_workspace_size_rejects_bad_shapes(L, args):
    assert ttq.ttq_workspace_size(*args, ttq.TTQ_BF16) == 0


def test_rejections_before_device_work(L):
    # unsupported bit width / group: refused before any CUDA call
    assert L.ttq_quantize_weight(None, 1, 4, 64, None, 5, 64, None, None, None, None, 0, None) == ttq.TTQ_ERR_UNSUPPORTED
    assert L.ttq_quantize_weight(None, 1, 4, 64, None, 4, 48, None, None, None, None, 0, None) == ttq.TTQ_ERR_UNSUPPORTED
    assert L.ttq_quantize_weight(None, 1, 4, 64, None, 0, 64, None, None, None, None, 0, None) == ttq.TTQ_ERR_INVALID_ARG
    # p < 1, lambda < 0, NaN alpha
    for p, lam, a in [(0.5, 0.0, 0.5), (2.0, -1.0, 0.5), (2.0, 0.0, float("nan"))]:
        st = L.ttq_act_norm(16, 1, 64, 4, p, lam, a, None, None, 256, 1 << 20, None)
        assert st == ttq.TTQ_ERR_INVALID_ARG
    # workspace too small / misaligned
    assert L.ttq_act_norm(16, 1, 64, 4, 2.0, 0.0, 0.5, None, None, 256, 64, None) == ttq.TTQ_ERR_WORKSPACE
    assert L.ttq_act_norm(16, 1, 64, 4, 2.0, 0.0, 0.5, None, None, 128, 1 << 20, None) == ttq.TTQ_ERR_INVALID_ARG
    # fused statistic + operand: Xs required, binary16 X refused, workspace checked
    assert L.ttq_act_norm_scale(16, 1, 64, 4, 2.0, 0.0, 0.5, None, None, None, 256, 1 << 20, None) == ttq.TTQ_ERR_INVALID_ARG
    assert L.ttq_act_norm_scale(16, 2, 64, 4, 2.0, 0.0, 0.5, None, None, 32, 256, 1 << 20, None) == ttq.TTQ_ERR_INVALID_ARG
    assert L.ttq_act_norm_scale(16, 1, 64, 4, 0.5, 0.0, 0.5, None, None, 32, 256, 1 << 20, None) == ttq.TTQ_ERR_INVALID_ARG
    assert L.ttq_act_norm_scale(16, 1, 64, 4, 2.0, 0.0, 0.5, None, None, 32, 256, 64, None) == ttq.TTQ_ERR_WORKSPACE
    assert L.ttq_act_norm_scale(16, 1, 64, 4, 2.0, 0.0, 0.5, None, None, 40, 256, 1 << 20, None) == ttq.TTQ_ERR_INVALID_ARG
    # dequantised-weight entry points: W_hat required, shapes checked before any CUDA call
    assert L.ttq_quantize_dequant_weight(16, 1, 4, 64, None, 4, 64, 16, 16, 16, None, 256, 4096, None) == ttq.TTQ_ERR_INVALID_ARG
    # codes, scales and zeros are given together, or all left out with W_hat given
    assert L.ttq_quantize_weight_ex(16, 1, 4, 64, None, 4, 64, 0, None, None, None, None, 256, 4096, None) == ttq.TTQ_ERR_INVALID_ARG
    assert L.ttq_quantize_weight_ex(16, 1, 4, 64, None, 4, 64, 0, 16, None, None, 16, 256, 4096, None) == ttq.TTQ_ERR_INVALID_ARG
    assert L.ttq_quantize_weight_ex(16, 1, 4, 64, None, 4, 64, 0, None, 16, 16, 16, 256, 4096, None) == ttq.TTQ_ERR_INVALID_ARG
    assert L.ttq_quantize_dequant_weight(16, 1, 4, 64, None, 5, 64, 16, 16, 16, 16, 256, 4096, None) == ttq.TTQ_ERR_UNSUPPORTED
    assert L.ttq_dequantized_gemm(16, 16, 60, 4, 4, 16, 1, 256, 4096, None) == ttq.TTQ_ERR_INVALID_ARG
    assert L.ttq_dequantized_gemm(16, None, 64, 4, 4, 16, 1, 256, 4096, None) == ttq.TTQ_ERR_INVALID_ARG
    assert L.ttq_dequantized_gemm(16, 16, 64, 4, 4, 16, 1, 256, 64, None) == ttq.TTQ_ERR_WORKSPACE
    assert L.ttq_dequantized_gemm(16, 16, 64, 4, 4, 16, 2, 256, 4096, None) == ttq.TTQ_ERR_INVALID_ARG
    # an unknown code scheme is refused before any CUDA call
    assert L.ttq_quantize_weight_ex(16, 1, 4, 64, None, 4, 64, 7, 16, 16, 16, None, 256, 4096, None) == ttq.TTQ_ERR_INVALID_ARG
    st = L.ttq_linear_forward_ex(16, 16, None, None, 1, 64, 64, 4, 0, 2.0, 0.0, 0.5, 4, 64, 9, 16, 1, 256, 1 << 30, None)
    assert st == ttq.TTQ_ERR_INVALID_ARG
    # forward with a null weight
    st = L.ttq_linear_forward(16, None, None, None, 1, 64, 64, 4, 0, 2.0, 0.0, 0.5, 4, 64, 16, 1, 256, 1 << 30, None)
    assert st == ttq.TTQ_ERR_INVALID_ARG
    assert L.ttq_workspace_init(None, 4096, None) == ttq.TTQ_ERR_INVALID_ARG
    assert L.ttq_get_status(None, None) == ttq.TTQ_ERR_INVALID_ARG


def test_lowrank_init_rejections_before_device_work(L):
    size = L.ttq_lowrank_workspace_size
    assert size(0, 64, 8, 8) == 0 and size(64, 64, 0, 8) == 0 and size(64, 64, 90, 8) == 0
    n = size(300, 200, 16, 8)
    assert n >= 4096 + 4 * 300 * 24 * 2 + 4 * 200 * 24
    init = L.ttq_lowrank_init
    ok = dict(W=16, dt=1, dp=300, d=200, r=16, ov=8, q=2, Om=32, B=48, A=64, R=80, ws=256, nb=n)

    def call(**kw):
        a = dict(ok, **kw)
        return init(a["W"], a["dt"], a["dp"], a["d"], a["r"], a["ov"], a["q"], a["Om"], a["B"], a["A"],
                    a["R"], a["ws"], a["nb"], None)

    assert call(dt=2) == ttq.TTQ_ERR_INVALID_ARG            # binary16 W
    assert call(r=0) == ttq.TTQ_ERR_INVALID_ARG
    assert call(ov=-1) == ttq.TTQ_ERR_INVALID_ARG
    assert call(q=17) == ttq.TTQ_ERR_INVALID_ARG
    assert call(r=90) == ttq.TTQ_ERR_UNSUPPORTED            # r + oversample > 96
    assert call(dp=20) == ttq.TTQ_ERR_UNSUPPORTED           # r + oversample > d'
    assert call(W=None) == ttq.TTQ_ERR_INVALID_ARG
    assert call(Om=None) == ttq.TTQ_ERR_INVALID_ARG
    assert call(A=72) == ttq.TTQ_ERR_INVALID_ARG            # not 16-byte aligned
    assert call(ws=128) == ttq.TTQ_ERR_INVALID_ARG          # not 256-byte aligned
    assert call(nb=n - 1) == ttq.TTQ_ERR_WORKSPACE


def test_fp8_scheme_rules_before_device_work(L):
    qw = L.ttq_quantize_weight_ex
    ASYM, SYM, FP8 = ttq.TTQ_QSCHEME_ASYMMETRIC, ttq.TTQ_QSCHEME_SYMMETRIC, ttq.TTQ_QSCHEME_FP8_E4M3
    # 8-bit codes only with the FP8 scheme, and FP8 only with 8 bits
    assert qw(16, 1, 4, 64, None, 8, 64, ASYM, 16, 16, 16, None, 256, 4096, None) == ttq.TTQ_ERR_UNSUPPORTED
    assert qw(16, 1, 4, 64, None, 8, 64, SYM, 16, 16, 16, None, 256, 4096, None) == ttq.TTQ_ERR_UNSUPPORTED
    assert qw(16, 1, 4, 64, None, 4, 64, FP8, 16, 16, 16, None, 256, 4096, None) == ttq.TTQ_ERR_UNSUPPORTED
    assert qw(16, 1, 4, 64, None, 8, 48, FP8, 16, 16, 16, None, 256, 4096, None) == ttq.TTQ_ERR_UNSUPPORTED
    assert qw(16, 1, 4, 64, None, 8, 64, 3, 16, 16, 16, None, 256, 4096, None) == ttq.TTQ_ERR_INVALID_ARG
    # 8-bit codes are read by the decode product only: at most 16 tokens,
    # d a multiple of 64
    st = L.ttq_dequant_gemm(16, 16, 16, None, 16, None, None, 1, 64, 64, 17, 0, 8, 64, 16, 1, 256, 1 << 30, None)
    assert st == ttq.TTQ_ERR_UNSUPPORTED
    st = L.ttq_dequant_gemm(16, 16, 16, None, 16, None, None, 1, 96, 64, 4, 0, 8, 32, 16, 1, 256, 1 << 30, None)
    assert st == ttq.TTQ_ERR_UNSUPPORTED
    # the default (asymmetric) forward refuses 8 bits; the FP8 forward checks its workspace
    st = L.ttq_linear_forward(16, 16, None, None, 1, 64, 64, 4, 0, 2.0, 0.0, 0.5, 8, 64, 16, 1, 256, 1 << 30, None)
    assert st == ttq.TTQ_ERR_UNSUPPORTED
    st = L.ttq_linear_forward_ex(16, 16, None, None, 1, 64, 64, 4, 0, 2.0, 0.0, 0.5, 8, 64, FP8, 16, 1, 256, 64,
                                 None)
    assert st == ttq.TTQ_ERR_WORKSPACE
    # FP8 layouts hold the binary16 W_hat beyond the decode product's reach
    # (T > 16); INT layouts only for T > 256
    for T, bits, present in [(4, 8, False), (1, 8, False), (16, 8, False), (17, 8, True),
                             (4, 4, False), (300, 4, True)]:
        lay = ttq.WorkspaceLayout()
        assert L.ttq_workspace_get_layout(256, 64, T, 0, bits, 64, 1, lay) == ttq.TTQ_OK
        assert (lay.wq != 0) == present, (T, bits)


def declared_arity():
    """Parameter count of every ttq_* function declared in the header."""
    text = re.sub(r"/\*.*?\*/", "", _header_text(), flags=re.S)
    out = {}
    for m in re.finditer(r"\b(ttq_[a-z_0-9]+)\s*\(([^;{]*?)\)\s*;", text):
        params = m.group(2).strip()
        out[m.group(1)] = 0 if params in ("", "void") else params.count(",") + 1
    return out


def test_binding_argument_counts_match_the_header():
    arity = declared_arity()
    assert set(arity) == set(ttq.SIGNATURES)
    for name, (_, argtypes) in ttq.SIGNATURES.items():
        assert len(argtypes) == arity[name], (name, len(argtypes), arity[name])
