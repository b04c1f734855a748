"""Pins of the TTQ oracle: checks against facts fixed outside the oracle.

Each check takes an ``Oracle`` instance and raises ``AssertionError`` when
the oracle disagrees with the fact it pins.  They are run on the real oracle
(tests/test_oracle.py) and on copies of it with a planted mistake, each of
which must fail at least one check (tests/test_oracle_mutants.py).

What pins what:
  hand worked example (tests/golden/hand_4x4.json) -> every step at once
  numpy float16 round-to-nearest + neighbour step  -> binary16 round-up
  numpy.linalg.norm and closed forms               -> the L_p statistic, D, D^{-1/2}
  brute force over all 2^b levels, exact ties      -> rounding and clamping of codes
  range / minimality properties of s and z         -> scale and zero point
  exact grids (idempotence), power-of-two scaling,
  row independence                                 -> quantiser and packing
  independent numpy unpack + dequant              -> bit layout and W_hat
  numpy matmul                                     -> Y and the low-rank term
"""
from __future__ import annotations

import json
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _f16_bits_to_f64(bits) -> np.ndarray:
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def _unpack_np(codes: np.ndarray, d: int, bits: int) -> np.ndarray:
    """Independent bit-stream reader: code i of a row is bits [b i, b i + b)
    of the row's little-endian uint32 words."""
    codes = np.asarray(codes, dtype=np.uint32)
    n = codes.shape[0]
    as_bytes = codes.view(np.uint8).reshape(n, -1)
    bitstream = np.unpackbits(as_bytes, axis=1, bitorder="little")
    idx = np.arange(d)[:, None] * bits + np.arange(bits)[None, :]
    sel = bitstream[:, idx]  # [n][d][bits]
    return (sel.astype(np.int64) << np.arange(bits)[None, None, :]).sum(axis=2)


def _dequant_np(codes, scales, zeros, Dr, d, bits, group) -> np.ndarray:
    q = _unpack_np(codes, d, bits).astype(np.float64)
    s = np.repeat(_f16_bits_to_f64(scales), group, axis=1)
    z = np.repeat(_f16_bits_to_f64(zeros), group, axis=1)
    dr = np.ones(d) if Dr is None else np.asarray(Dr, np.float64)
    return s * (q - z) * dr[None, :]


def _rand_weights(rng, dp, d, std=0.05):
    return (rng.standard_normal((dp, d)) * std).astype(np.float32)


# --------------------------------------------------------------------------
def check_hand_example(O):
    g = json.load(open(os.path.join(GOLDEN, "hand_4x4.json")))
    pr = g["params"]
    X = np.array(g["X"], np.float64)
    W = np.array(g["W"], np.float32)
    out = O.forward(X, W, pr["p"], pr["lambda"], pr["alpha"], pr["bits"], pr["group"])
    assert out["status"] == 0, out["status"]
    assert np.array_equal(out["D"], np.array(g["D"], np.float64)), out["D"]
    assert np.array_equal(out["Dr"], np.array(g["D_rsqrt"], np.float64)), out["Dr"]
    assert np.array_equal(out["codes"].ravel(), np.array(g["packed_words"], np.uint32)), out["codes"]
    assert np.array_equal(O.unpack(out["codes"], 4, pr["bits"]), np.array(g["codes"])), "unpack"
    assert np.array_equal(out["scales"].ravel(), np.array(g["scales_f16_bits"], np.uint16)), out["scales"]
    assert np.array_equal(out["zeros"].ravel(), np.array(g["zeros_f16_bits"], np.uint16)), out["zeros"]
    What = O.dequant_rows(out["codes"], out["scales"], out["zeros"], out["Dr"], 4, pr["bits"], pr["group"])
    assert np.array_equal(What, np.array(g["W_hat"], np.float64)), What
    assert np.array_equal(out["Y"], np.array(g["Y"], np.float64)), out["Y"]


def check_f16_round_up(O):
    """binary16 rounding toward +inf, against numpy's nearest-even float16
    conversion moved one step up whenever it landed below the input."""
    pats = np.arange(0, 0x10000, dtype=np.uint32).astype(np.uint16)
    h = pats.view(np.float16)
    h = h[np.isfinite(h)].astype(np.float32)
    cand = [h, np.nextafter(h, np.float32(np.inf)), np.nextafter(h, np.float32(-np.inf))]
    rng = np.random.default_rng(7)
    cand.append(rng.uniform(-70000, 70000, 20000).astype(np.float32))
    cand.append((rng.uniform(-1, 1, 20000) * 2.0 ** rng.integers(-30, -10, 20000)).astype(np.float32))
    cand.append(np.array([65504, 65505, 65519, 65520, 1e9, -65504, -65505, -65520, -1e9, 0.0, -0.0,
                          2 ** -24, 2 ** -25, 3 * 2 ** -26, 2 ** -14, 2 ** -14 * 1.0001], np.float32))
    v = np.concatenate(cand)
    with np.errstate(over="ignore"):
        near = v.astype(np.float16)
        below = near.astype(np.float32) < v
        up = near.copy()
        up[below] = np.nextafter(near[below], np.float16(np.inf))
    expect = up.view(np.uint16)
    got = np.fromiter((O.lib.ttqo_f32_to_f16_ru(float(x)) for x in v), dtype=np.uint16, count=v.size)
    bad = np.nonzero(got != expect)[0]
    assert bad.size == 0, f"{bad.size} mismatches, first x={v[bad[0]]!r} got {got[bad[0]]:#06x} want {expect[bad[0]]:#06x}"


def check_f16_decode(O):
    pats = np.arange(0, 0x10000, dtype=np.uint32).astype(np.uint16)
    ref = pats.view(np.float16).astype(np.float32)
    got = np.fromiter((O.lib.ttqo_f16_to_f32(int(p)) for p in pats), dtype=np.float32, count=pats.size)
    ok = (got == ref) | (np.isnan(got) & np.isnan(ref))
    assert ok.all(), np.nonzero(~ok)[0][:5]


def check_act_norm(O):
    rng = np.random.default_rng(11)
    T, d = 37, 24
    X = rng.standard_normal((T, d)) * np.exp(rng.uniform(-3, 3, d))[None, :]
    for p in (1.0, 2.0, 3.0):
        n = np.linalg.norm(X, ord=p, axis=0)
        D, Dr, st = O.act_norm(X, p, 0.0, 1.0)
        assert st == 0
        assert np.allclose(D, n, rtol=1e-12, atol=0), (p, D, n)
        assert np.allclose(D * Dr * Dr, 1.0, rtol=1e-14, atol=0)
        D0, Dr0, st = O.act_norm(X, p, 0.3, 0.0)
        assert st == 0 and np.array_equal(D0, np.ones(d)) and np.array_equal(Dr0, np.ones(d))
        Dh, _, _ = O.act_norm(X, p, 0.25, 0.5)
        assert np.allclose(Dh * Dh, n + 0.25, rtol=1e-12, atol=0), p
        D3, _, _ = O.act_norm(X, p, 0.5, 3.0)
        assert np.allclose(D3, (n + 0.5) ** 3, rtol=1e-12, atol=0), p
    # constant channels: ||c 1_T||_p = |c| T^(1/p)
    c = np.array([0.0, 1.0, -2.5, 1e-3, 7.0, -64.0])
    Xc = np.tile(c, (T, 1))
    for p in (1.0, 2.0, 4.0):
        D, _, _ = O.act_norm(Xc, p, 0.0, 1.0)
        assert np.allclose(D, np.abs(c) * T ** (1.0 / p), rtol=1e-13, atol=0), p
    # a zero channel with lambda = 0 gives D = 0: flagged
    _, _, st = O.act_norm(Xc, 2.0, 0.0, 0.5)
    assert st & 4, st


def _grid_case(rng, dp, d, bits, group, with_ties=False):
    """W on an exact quantisation grid: per group s = 2^e, z in [0, qmax],
    codes spanning both ends.  Returns W, s, z, q."""
    qmax = (1 << bits) - 1
    ng = d // group
    e = rng.integers(-9, 3, (dp, ng))
    s = np.ldexp(1.0, e)
    z = rng.integers(0, qmax + 1, (dp, ng))
    q = rng.integers(0, qmax + 1, (dp, d))
    for j in range(dp):
        for k in range(ng):
            a, b = rng.choice(group, 2, replace=False)
            q[j, k * group + a] = 0
            q[j, k * group + b] = qmax
    sr = np.repeat(s, group, axis=1)
    zr = np.repeat(z, group, axis=1)
    W = (sr * (q - zr)).astype(np.float32)
    return W, s, z, q


def check_exact_grid(O):
    """Quantising an exactly representable grid returns it unchanged
    (idempotence), with the grid's own scale, zero and codes."""
    rng = np.random.default_rng(5)
    for bits in (2, 3, 4, 8):
        for group in (32, 64):
            dp, d = 6, 128
            W, s, z, q = _grid_case(rng, dp, d, bits, group)
            codes, sc, ze, st = O.quantize(W, None, bits, group)
            assert st == 0
            assert np.array_equal(_f16_bits_to_f64(sc), s), (bits, group)
            assert np.array_equal(_f16_bits_to_f64(ze), z.astype(np.float64)), (bits, group)
            assert np.array_equal(_unpack_np(codes, d, bits), q), (bits, group)
            What = O.dequant_rows(codes, sc, ze, None, d, bits, group)
            assert np.array_equal(What, W.astype(np.float64)), (bits, group)
            assert np.array_equal(What, _dequant_np(codes, sc, ze, None, d, bits, group))
            # with D = 4^k the pre-scale is an exact power of two, undone by D^{-1/2}
            kexp = rng.integers(-3, 4, d)
            D = np.ldexp(1.0, 2 * kexp).astype(np.float32)
            Wd = (W / np.ldexp(1.0, kexp)[None, :]).astype(np.float32)
            codes2, sc2, ze2, st = O.quantize(Wd, D, bits, group)
            assert st == 0
            assert np.array_equal(codes2, codes) and np.array_equal(sc2, sc) and np.array_equal(ze2, ze)
            Dr = 1.0 / np.sqrt(D.astype(np.float64))
            assert np.array_equal(O.dequant_rows(codes2, sc2, ze2, Dr, d, bits, group), Wd.astype(np.float64))


def check_ties_even(O):
    """Exact half-way points round to the even level (rint), both signs."""
    bits, group = 4, 32
    row = np.zeros(32, np.float32)
    # range [0, 15] -> s = 1, z = 0; ties at 0.5 .. 6.5
    row[0], row[1] = 0.0, 15.0
    row[2:9] = np.array([0.5, 1.5, 2.5, 3.5, 4.5, 5.5, 6.5], np.float32)
    # second row: range [-7.5, 7.5] -> s = 1, z = rint(7.5) = 8
    row2 = np.zeros(32, np.float32)
    row2[0], row2[1] = -7.5, 7.5
    row2[2:8] = np.array([-0.5, -1.5, -2.5, 0.5, 1.5, 2.5], np.float32)
    codes, sc, ze, st = O.quantize(np.stack([row, row2]), None, bits, group)
    q = _unpack_np(codes, 32, bits)
    assert _f16_bits_to_f64(sc).tolist() == [[1.0], [1.0]], sc
    assert _f16_bits_to_f64(ze).tolist() == [[0.0], [8.0]], ze
    assert q[0, 2:9].tolist() == [0, 2, 2, 4, 4, 6, 6], q[0]
    # rint(-7.5) = -8 -> 0 ; rint(7.5) = 8 -> 16 -> clamped to 15
    assert q[1, 0] == 0 and q[1, 1] == 15, q[1]
    assert q[1, 2:8].tolist() == [8, 6, 6, 8, 10, 10], q[1]


def check_code_rounding_exact_product(O):
    """The code rounds the exact product x * (1/s), not its binary32 rounding.
    Group [0, 45] gives s = 3 and z = 0, inv = binary32(1/3).  For x =
    28.499998092651367 the binary32 product is exactly 9.5 (rint: 10) while
    the true product is 9.49999964... (rint: 9); x = 28.5 is a control."""
    bits, group = 4, 32
    row = np.zeros(32, np.float32)
    row[0], row[1] = 0.0, 45.0
    x_tie = np.float32(28.499998092651367)
    row[2], row[3] = x_tie, 28.5
    inv = np.float32(1.0) / np.float32(3.0)
    assert np.float32(x_tie * inv) == np.float32(9.5)            # the binary32 product is a tie
    assert float(x_tie) * float(inv) < 9.5                       # the true one is below it
    codes, sc, ze, st = O.quantize(row[None, :], None, bits, group)
    assert st == 0
    assert _f16_bits_to_f64(sc).tolist() == [[3.0]] and _f16_bits_to_f64(ze).tolist() == [[0.0]]
    q = _unpack_np(codes, 32, bits)
    assert q[0, 1] == 15 and q[0, 2] == 9 and q[0, 3] == 10, q[0, :4]


def check_symmetric_worked_example(O):
    """The symmetric INT4 quantiser on the blog's group ("The maths that
    matter"): magnitudes 1 with one 30 give s = 30/7 (here the binary16 value
    just above it) and errors up to s/2 ~ 2.14 on the unit values; without
    the 30 the scale is 1/7 and the errors at most ~0.071, thirty times
    less.  Levels are +-7 around the stored zero point 8."""
    g = json.load(open(os.path.join(GOLDEN, "blog_int4_outlier.json")))["printed"]
    bits, group = 4, 32
    row = np.ones(32, np.float32)
    row[1::2] = -1.0
    row[5] = 30.0
    codes, sc, ze, st = O.quantize(row[None, :], None, bits, group, symmetric=True)
    assert st == 0
    s = float(_f16_bits_to_f64(sc)[0, 0])
    assert 30.0 / 7.0 <= s <= 30.0 / 7.0 * (1 + 2.0 ** -10), s
    assert _f16_bits_to_f64(ze).tolist() == [[8.0]]
    q = _unpack_np(codes, 32, bits)[0]
    assert q[5] == 15 and q.min() >= 1 and q.max() <= 15
    rec = s * (q.astype(np.float64) - 8.0)
    unit_err = np.abs(rec - row)[np.arange(32) != 5]
    assert unit_err.max() <= s / 2 and abs(s / 2 - 2.1428571) < 2e-3, (unit_err.max(), s)
    # the values the page prints, to their printed digits
    assert abs(s - g["shared_scale"]) <= 0.005 and abs(s / 2 - g["shared_max_error_typical"]) <= 0.005
    assert abs(s / 2 / 1.0 - g["shared_relative_error_typical"]) <= 0.005
    # segregated: the same unit values without the outlier
    row2 = row.copy()
    row2[5] = 1.0
    codes2, sc2, _, _ = O.quantize(row2[None, :], None, bits, group, symmetric=True)
    s2 = float(_f16_bits_to_f64(sc2)[0, 0])
    assert 1.0 / 7.0 <= s2 <= 1.0 / 7.0 * (1 + 2.0 ** -10), s2
    err2 = np.abs(s2 * (_unpack_np(codes2, 32, bits)[0] - 8.0) - row2)
    assert err2.max() <= s2 / 2 and abs(s2 / 2 - 0.0714286) < 1e-4
    assert abs(s2 - g["segregated_scale"]) <= 0.0005 and abs(s2 / 2 - g["segregated_max_error_typical"]) <= 0.0005
    assert abs(s2 / 2 - g["segregated_relative_error_typical"]) <= 0.005
    assert abs(s / s2 - g["error_ratio"]) <= 0.5
    # the asymmetric quantiser on the outlier group: s = (30 - m) / 15, m = -1
    codes3, sc3, ze3, _ = O.quantize(row[None, :], None, bits, group)
    s3 = float(_f16_bits_to_f64(sc3)[0, 0])
    assert 31.0 / 15.0 <= s3 <= 31.0 / 15.0 * (1 + 2.0 ** -10)
    rec3 = s3 * (_unpack_np(codes3, 32, bits)[0] - _f16_bits_to_f64(ze3)[0, 0])
    assert np.abs(rec3 - row).max() <= s3 / 2 * (1 + 1e-6)


def check_symmetric_properties(O):
    """Symmetric quantiser: codes in [1, 2^b - 1], zero point 2^(b-1), every
    element within s/2, the nearest of the 2^b - 1 levels (ties to even),
    s the smallest binary16 covering max|x| (or the 2^-14 floor), and odd
    symmetry: -W gives the mirrored codes."""
    rng = np.random.default_rng(11)
    for bits in (2, 3, 4):
        for group in (32, 128):
            dp, d = 8, 256
            W = _rand_weights(rng, dp, d)
            W[0, :group] = 0.0
            D = np.exp(rng.uniform(-3, 3, d)).astype(np.float32)
            codes, sc, ze, st = O.quantize(W, D, bits, group, symmetric=True)
            assert st == 0
            lmax = (1 << (bits - 1)) - 1
            zero = 1 << (bits - 1)
            q = _unpack_np(codes, d, bits)
            assert q.min() >= 1 and q.max() <= 2 * lmax + 1, (bits, group)
            assert np.all(_f16_bits_to_f64(ze) == zero)
            x = (W.astype(np.float32) * np.sqrt(D).astype(np.float32)[None, :]).astype(np.float64)
            s = np.repeat(_f16_bits_to_f64(sc), group, axis=1)
            lev = q.astype(np.float64) - zero
            err = np.abs(x - s * lev)
            assert np.all(err <= s / 2 * (1 + 1e-6)), (bits, group)
            levels = np.arange(-lmax, lmax + 1)[None, None, :]
            dist = np.abs(x[:, :, None] - s[:, :, None] * levels)
            best = dist.min(axis=2)
            near_tie = np.abs(np.abs(x / s - np.round(x / s)) - 0.5) < 1e-5
            assert np.all((err <= best * (1 + 1e-9) + 1e-300) | near_tie), (bits, group)
            M = np.abs(x).reshape(dp, d // group, group).max(axis=2)
            s16 = sc.view(np.float16)
            sv = s16.astype(np.float64)
            floor_ok = sv == 2.0 ** -14
            assert np.all(sv * lmax >= M * (1 - 2.0 ** -22))
            below = np.nextafter(s16, np.float16(0)).astype(np.float64)
            assert np.all(floor_ok | (below * lmax < M * (1 + 2.0 ** -22))), (bits, group)
            codes_n, sc_n, _, _ = O.quantize(-W, D, bits, group, symmetric=True)
            assert np.array_equal(sc_n, sc)
            assert np.array_equal(_unpack_np(codes_n, d, bits), 2 * zero - q), (bits, group)


def check_quantizer_properties(O):
    """Codes in range; per-element error <= s/2 (+ reciprocal slack); the
    stored scale is the smallest binary16 value covering the group range;
    zeros are integers in range; brute force over all levels agrees."""
    rng = np.random.default_rng(3)
    for bits in (2, 3, 4):
        for group in (32, 64, 128):
            dp, d = 8, 256
            W = _rand_weights(rng, dp, d)
            W[0, :group] = 0.0                    # degenerate group
            W[1, :group] = np.abs(W[1, :group])   # one-signed group
            D = np.exp(rng.uniform(-4, 4, d)).astype(np.float32)
            codes, sc, ze, st = O.quantize(W, D, bits, group)
            assert st == 0
            qmax = (1 << bits) - 1
            q = _unpack_np(codes, d, bits)
            assert q.min() >= 0 and q.max() <= qmax
            x = W.astype(np.float32) * np.sqrt(D).astype(np.float32)[None, :]
            s = np.repeat(_f16_bits_to_f64(sc), group, axis=1)
            z = np.repeat(_f16_bits_to_f64(ze), group, axis=1)
            assert np.all(z == np.round(z)) and z.min() >= 0 and z.max() <= qmax
            err = np.abs(x.astype(np.float64) - s * (q - z))
            slack = 2.0 ** -20 * np.abs(x).max()
            assert np.all(err <= s / 2 + slack), (bits, group, (err - s / 2).max())
            # scale: s >= range/qmax, and the binary16 value just below is not
            xg = x.reshape(dp, d // group, group).astype(np.float64)
            rng_ = np.maximum(xg.max(axis=2), 0) - np.minimum(xg.min(axis=2), 0)
            s16 = sc.view(np.float16)
            sv = s16.astype(np.float64)
            assert np.all(sv * qmax >= rng_ * (1 - 2.0 ** -22)), (bits, group)
            below = np.nextafter(s16, np.float16(0)).astype(np.float64)
            floor_ok = sv == 2.0 ** -14
            assert np.all(floor_ok | (below * qmax < rng_ * (1 + 2.0 ** -22))), (bits, group)
            assert np.all(floor_ok[:1, 0]), "degenerate group must take the 2^-14 floor"
            # brute force: the nearest level, ties to the even rint result
            levels = np.arange(qmax + 1)[None, None, :]
            dist = np.abs(x.astype(np.float64)[:, :, None] - s[:, :, None] * (levels - z[:, :, None]))
            best = dist.min(axis=2)
            mine = np.take_along_axis(dist, q[:, :, None], axis=2)[:, :, 0]
            near_tie = np.abs(np.abs(x / s - np.round(x / s)) - 0.5) < 1e-5
            assert np.all((mine <= best * (1 + 1e-9) + 1e-300) | near_tie), (bits, group)


def check_scaling_and_rows(O):
    """W * 2^k scales s by 2^k and keeps codes and zeros; any subset of rows
    quantises to the same bits; D computed with alpha = 0 is the identity
    (TTQ reduces to plain round-to-nearest)."""
    rng = np.random.default_rng(9)
    dp, d, bits, group = 12, 256, 3, 64
    W = _rand_weights(rng, dp, d, 0.5)
    D = np.exp(rng.uniform(-2, 2, d)).astype(np.float32)
    codes, sc, ze, _ = O.quantize(W, D, bits, group)
    for k in (-3, 2):
        c2, s2, z2, _ = O.quantize((W * np.float32(2.0 ** k)).astype(np.float32), D, bits, group)
        assert np.array_equal(c2, codes) and np.array_equal(z2, ze)
        assert np.array_equal(_f16_bits_to_f64(s2), _f16_bits_to_f64(sc) * 2.0 ** k)
    rows = np.array([0, 5, 6, 11])
    c3, s3, z3, _ = O.quantize(W[rows], D, bits, group)
    assert np.array_equal(c3, codes[rows]) and np.array_equal(s3, sc[rows]) and np.array_equal(z3, ze[rows])
    X = rng.standard_normal((5, d))
    D0, _, _ = O.act_norm(X, 2.0, 1e-3, 0.0)
    a = O.quantize(W, D0.astype(np.float32), bits, group)
    b = O.quantize(W, None, bits, group)
    assert all(np.array_equal(u, v) for u, v in zip(a[:3], b[:3]))


def check_dequant_layout(O):
    """W_hat = s (q - z) D^{-1/2} read back through an independent unpacker."""
    rng = np.random.default_rng(13)
    for bits in (2, 3, 4):
        dp, d, group = 5, 192, 64
        W = _rand_weights(rng, dp, d)
        D = np.exp(rng.uniform(-2, 2, d))
        codes, sc, ze, _ = O.quantize(W, D.astype(np.float32), bits, group)
        Dr = 1.0 / np.sqrt(D)
        ref = _dequant_np(codes, sc, ze, Dr, d, bits, group)
        got = O.dequant_rows(codes, sc, ze, Dr, d, bits, group)
        assert np.array_equal(got, ref), bits
        rows = np.array([4, 1])
        assert np.array_equal(O.dequant_rows(codes, sc, ze, Dr, d, bits, group, rows), ref[rows])


def check_projection(O):
    """Y = W_hat X and the low-rank term against numpy fp64 matmuls."""
    rng = np.random.default_rng(17)
    T, d, dp, r = 9, 64, 7, 5
    X = rng.standard_normal((T, d))
    W = _rand_weights(rng, dp, d)
    A = rng.standard_normal((r, d)) * 0.1
    B = rng.standard_normal((dp, r)) * 0.1
    out = O.forward(X, W, 2.0, 1e-3, 0.5, 4, 32)
    What = O.dequant_rows(out["codes"], out["scales"], out["zeros"], out["Dr"], d, 4, 32)
    ref = X @ What.T
    assert np.allclose(out["Y"], ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    out2 = O.forward(X, W, 2.0, 1e-3, 0.5, 4, 32, A=A, B=B)
    ref2 = ref + (X @ A.T) @ B.T
    assert np.allclose(out2["Y"], ref2, rtol=1e-12, atol=1e-12 * np.abs(ref2).max())
    rows = np.array([6, 0, 3])
    out3 = O.forward(X, W, 2.0, 1e-3, 0.5, 4, 32, A=A, B=B, rows=rows)
    assert np.allclose(out3["Y"], ref2[:, rows], rtol=1e-12, atol=1e-12 * np.abs(ref2).max())


def check_x_rescale(O):
    """With alpha = 0 any rescaling of X leaves W_hat unchanged; with
    lambda = 0, alpha = 1, p = 1, X * 16 gives D * 16 and sqrt(D) * 4
    exactly: the codes are unchanged and Y scales by exactly 16."""
    rng = np.random.default_rng(19)
    T, d, dp = 6, 64, 4
    X = rng.standard_normal((T, d))
    W = _rand_weights(rng, dp, d)
    a = O.forward(X, W, 2.0, 1e-3, 0.0, 4, 32)
    b = O.forward(X * 123.25, W, 2.0, 1e-3, 0.0, 4, 32)
    assert np.array_equal(a["codes"], b["codes"]) and np.array_equal(a["scales"], b["scales"])
    c = O.forward(X, W, 1.0, 0.0, 1.0, 4, 32)
    e = O.forward(X * 16.0, W, 1.0, 0.0, 1.0, 4, 32)
    assert np.array_equal(e["D"], c["D"] * 16.0)
    assert np.array_equal(c["codes"], e["codes"]) and np.array_equal(c["zeros"], e["zeros"])
    assert np.array_equal(_f16_bits_to_f64(e["scales"]), _f16_bits_to_f64(c["scales"]) * 4.0)
    assert np.array_equal(e["Y"], c["Y"] * 16.0)


def check_nonfinite(O):
    W = np.zeros((2, 32), np.float32)
    W[1, 3] = np.nan
    _, _, _, st = O.quantize(W, None, 4, 32)
    assert st & 4
    W2 = np.zeros((1, 32), np.float32)
    W2[0, 0] = 1e6  # scale (1e6 / 15) exceeds binary16
    _, sc, _, st = O.quantize(W2, None, 4, 32)
    assert st & 4 and sc[0, 0] == 0x7C00


def check_method_effect(O):
    """The effect the pages claim: with outlier channels in X, the
    activation-aware W_hat (alpha = 0.5) reconstructs W X better than plain
    round-to-nearest (alpha = 0)."""
    rng = np.random.default_rng(23)
    T, d, dp = 32, 256, 64
    X = rng.standard_normal((T, d))
    X[:, rng.choice(d, 4, replace=False)] *= 50.0
    W = _rand_weights(rng, dp, d, 0.02)
    ref = X @ W.astype(np.float64).T
    e_ttq = np.linalg.norm(O.forward(X, W, 2.0, 1e-3, 0.5, 3, 64)["Y"] - ref)
    e_rtn = np.linalg.norm(O.forward(X, W, 2.0, 1e-3, 0.0, 3, 64)["Y"] - ref)
    assert e_ttq < 0.8 * e_rtn, (e_ttq, e_rtn)


# ---------------------------------------------------------------- FP8 codes
# E4M3 as the OCP 8-bit floating point specification defines it: sign,
# 4 exponent bits with bias 7, 3 fraction bits, subnormals at exponent 0,
# no infinities, S.1111.111 NaN, largest finite 448.  The values below are
# written out from that definition (not produced by the oracle).
_E4M3_KNOWN = {0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0x30: 0.5,
               0x38: 1.0, 0x39: 1.125, 0x3C: 1.5, 0x40: 2.0, 0x44: 3.0, 0x6C: 96.0, 0x6D: 104.0,
               0x77: 240.0, 0x78: 256.0, 0x7E: 448.0, 0x80: -0.0, 0xB8: -1.0, 0xFE: -448.0}


def _e4m3_by_definition(code: int) -> float:
    e, m = (code >> 3) & 15, code & 7
    if e == 15 and m == 7:
        return float("nan")
    v = m / 8 * 2.0 ** -6 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7)
    return -v if code & 0x80 else v


def check_e4m3_table(O):
    for c, v in _E4M3_KNOWN.items():
        got = O.e4m3_value(c)
        assert got == v and np.signbit(got) == np.signbit(v), (hex(c), got, v)
    for c in range(256):
        want = _e4m3_by_definition(c)
        got = O.e4m3_value(c)
        assert (np.isnan(want) and np.isnan(got)) or got == want, (hex(c), got, want)
    finite = [O.e4m3_value(c) for c in range(0x7F)]
    assert all(b > a for a, b in zip(finite, finite[1:]))          # monotone in the code
    assert sum(np.isnan(O.e4m3_value(c)) for c in range(256)) == 2  # 0x7F and 0xFF


def check_e4m3_rounding(O):
    vals = [_e4m3_by_definition(c) for c in range(0x7F)]
    for c in range(0x7E):
        a, b = vals[c], vals[c + 1]
        mid = (a + b) / 2
        even = c if c % 2 == 0 else c + 1
        assert O.e4m3_from(mid) == even, (hex(c), mid)              # ties to the even code
        assert O.e4m3_from(mid * (1 - 2.0 ** -30)) == c
        assert O.e4m3_from(mid * (1 + 2.0 ** -30)) == c + 1
        assert O.e4m3_from(-b) == (c + 1) | 0x80
    for big in (448.0, 460.0, 464.0, 500.0, 1e30):
        assert O.e4m3_from(big) == 0x7E and O.e4m3_from(-big) == 0xFE
    assert O.e4m3_from(-0.0) == 0x80 and O.e4m3_from(2.0 ** -11) == 0x00
    assert O.e4m3_from(-(2.0 ** -10) * 1.5) == 0x81                 # nearer 2^-9 than 0


def check_fp8_worked_example(O):
    # one group of 8, D = I: the group's largest magnitude is 448, so s = 1
    # and each code is the E4M3 rounding of the weight itself (100 lies
    # half-way between 96 and 104 and goes to the even code, 96)
    row = np.array([[0.0, 1.0, 2.0, 3.0, 448.0, -448.0, 0.5, 100.0]], np.float32)
    codes, sc, ze, st = O.quantize_fp8(row, None, 8)
    assert st == 0
    assert sc.tolist() == [[0x3C00]] and ze.tolist() == [[0]]
    assert codes.tolist() == [[0x44403800, 0x6C30FE7E]], [hex(x) for x in codes.ravel()]
    What = O.dequant_rows_fp8(codes, sc, None, 8, 8)
    assert What.tolist() == [[0.0, 1.0, 2.0, 3.0, 448.0, -448.0, 0.5, 96.0]]


def check_fp8_properties(O):
    g = np.random.Generator(np.random.PCG64(77))
    d, group = 256, 64
    W = (g.standard_normal((6, d)) * 0.05).astype(np.float32)
    W[:, 17] *= 60.0
    D = np.exp(g.uniform(-3, 3, d)).astype(np.float32)
    codes, sc, ze, st = O.quantize_fp8(W, D, group)
    assert st == 0 and not ze.any()
    q = codes.view(np.uint8).reshape(6, d)                       # bytes in code order
    s = _f16_bits_to_f64(sc)
    x = W.astype(np.float64) * np.sqrt(D.astype(np.float64))
    vals = np.vectorize(_e4m3_by_definition)(q.astype(np.int64))
    rec = np.repeat(s, group, axis=1) * vals
    sg = np.repeat(s, group, axis=1)
    # 3 fraction bits: half an ulp is 2^-4 relative in the normal range,
    # 2^-10 s absolute among the subnormals (plus binary32 slack)
    assert np.all(np.abs(rec - x) <= 2.0 ** -4 * np.abs(x) * (1 + 1e-5) + 2.0 ** -10 * sg * (1 + 1e-5))
    # the oracle's reconstruction s e4m3(q) D^-1/2 against the same
    # statement in numpy (scales far from 1, D^-1/2 far from 1)
    Dr = 1.0 / np.sqrt(D.astype(np.float64))
    What = O.dequant_rows_fp8(codes, sc, Dr, d, group)
    assert np.max(np.abs(What - rec * Dr)) <= 1e-12 * np.max(np.abs(rec * Dr))
    # every group's largest magnitude is coded as +-448
    for j in range(6):
        for k in range(d // group):
            blk = x[j, k * group:(k + 1) * group]
            i = int(np.argmax(np.abs(blk)))
            assert q[j, k * group + i] & 0x7F == 0x7E
    # odd symmetry: -W flips exactly the sign bit of every code
    codes_n, sc_n, _, _ = O.quantize_fp8(-W, D, group)
    assert np.array_equal(sc_n, sc)
    assert np.array_equal(codes_n.view(np.uint8), codes.view(np.uint8) ^ 0x80)


ALL_CHECKS = [
    check_hand_example,
    check_f16_round_up,
    check_f16_decode,
    check_act_norm,
    check_exact_grid,
    check_ties_even,
    check_code_rounding_exact_product,
    check_symmetric_worked_example,
    check_symmetric_properties,
    check_quantizer_properties,
    check_scaling_and_rows,
    check_dequant_layout,
    check_e4m3_table,
    check_e4m3_rounding,
    check_fp8_worked_example,
    check_fp8_properties,
    check_projection,
    check_x_rescale,
    check_nonfinite,
    check_method_effect,
]
