"""Planted mistakes: each edited copy of the oracle must fail a pin.

A plausible slip anywhere in the oracle -- a dropped term, a wrong sign,
exponent or index, another rounding rule, a transposed operand -- is
planted in a copy of its C source (on the CPU only), compiled, and run
against every pin in a child process.  The pins are adequate only if every
such copy fails at least one of them.
"""
import os
import subprocess
import sys

import pytest

import ttq_oracle

HERE = os.path.dirname(os.path.abspath(__file__))

# (name, text in the oracle source, replacement)
MUTANTS = [
    ("sqrt_of_D_dropped", "h[i] = D ? sqrtf(D[i]) : 1.0f;", "h[i] = D ? D[i] : 1.0f;"),
    ("prescale_divides", "x[c] = w * h[i];", "x[c] = w / h[i];"),
    ("range_without_zero", "float m = 0.0f, M = 0.0f;", "float m = 3e38f, M = -3e38f;"),
    ("levels_off_by_one", "float s32 = range / (float)qmax;", "float s32 = range / (float)(qmax + 1);"),
    ("scale_floor_dropped", "float s32 = range / (float)qmax;\n      if (!(s32 >= 0x1p-14f)) s32 = 0x1p-14f;",
     "float s32 = range / (float)qmax;"),
    ("sym_scale_floor_dropped", "if (!(s32 >= 0x1p-14f)) s32 = 0x1p-14f; /* binary16 normal range */", ""),
    ("codes_floor_not_rint", "double r = rint((double)x[c] * (double)inv);",
     "double r = floor((double)x[c] * (double)inv);"),
    ("codes_half_away", "double r = rint((double)x[c] * (double)inv);",
     "double r = round((double)x[c] * (double)inv);"),
    ("codes_product_rounded_first", "double r = rint((double)x[c] * (double)inv);",
     "double r = rint((double)(x[c] * inv));"),
    ("sym_levels_unsigned", "const int lmax = (1 << (bits - 1)) - 1;", "const int lmax = (1 << bits) - 1;"),
    ("sym_range_signed_max", "float a = fabsf(v[c]);", "float a = v[c];"),
    ("sym_prescale_divides", "v[c] = w * sq[i];", "v[c] = w / sq[i];"),
    ("sym_codes_floor", "long l = (long)rint((double)v[c] * (double)inv);",
     "long l = (long)floor((double)v[c] * (double)inv);"),
    ("sym_zero_dropped", "zeros[j * ngroups + k] = f16_from_small_int(zero);",
     "zeros[j * ngroups + k] = f16_from_small_int(0);"),
    ("zero_sign_flipped", "double zr = rint(-(double)m * (double)inv);",
     "double zr = rint((double)m * (double)inv);"),
    ("zero_point_subtracted", "long q = (long)r + z;", "long q = (long)r - z;"),
    ("min_tracks_max", "if (x[c] < m) m = x[c];", "if (x[c] > m) m = x[c];"),
    ("scale_round_nearest", "double n = sign ? floor(m) : ceil(m);", "double n = nearbyint(m);"),
    ("scale_round_down", "double n = sign ? floor(m) : ceil(m);", "double n = sign ? ceil(m) : floor(m);"),
    ("f16_exponent_bias", "v = ldexp(1024.0 + (double)f, e - 25);", "v = ldexp(1024.0 + (double)f, e - 24);"),
    ("norm_root_dropped", "double n = pow(acc, 1.0 / p);", "double n = acc;"),
    ("norm_mean_not_sum", "double n = pow(acc, 1.0 / p);", "double n = pow(acc / (double)(T > 0 ? T : 1), 1.0 / p);"),
    ("alpha_dropped", "double Di = pow(n + lambda, alpha);", "double Di = n + lambda;"),
    ("lambda_dropped", "double Di = pow(n + lambda, alpha);", "double Di = pow(n, alpha);"),
    ("Dr_wrong_power", "Dr[i] = 1.0 / sqrt(Di);", "Dr[i] = 1.0 / Di;"),
    ("dequant_adds_zero", "What[rr * d + i] = s * (q - z) * dr;", "What[rr * d + i] = s * (q + z) * dr;"),
    ("dequant_keeps_prescale", "What[rr * d + i] = s * (q - z) * dr;", "What[rr * d + i] = s * (q - z);"),
    ("dequant_wrong_group", "int64_t k = i / group;", "int64_t k = (i / group + 1) % ngroups;"),
    ("pack_msb_first", "if ((q >> k) & 1u) row[bit >> 5] |= 1u << (bit & 31);",
     "if ((q >> (bits - 1 - k)) & 1u) row[bit >> 5] |= 1u << (bit & 31);"),
    ("project_channel_reversed", "acc += What[r * d + i] * X[t * d + i];",
     "acc += What[r * d + i] * X[t * d + (d - 1 - i)];"),
    ("lowrank_dropped", "Y[t * nrows + r] += acc;", "Y[t * nrows + r] += 0.0 * acc;"),
    ("e4m3_exponent_bias", "else v = ldexp(8.0 + (double)m, e - 10);", "else v = ldexp(8.0 + (double)m, e - 11);"),
    ("e4m3_subnormal_scale", "if (e == 0) v = ldexp((double)m, -9);", "if (e == 0) v = ldexp((double)m, -10);"),
    ("e4m3_nan_code", "if (e == 15 && m == 7) return NAN;", "if (e == 15 && m == 6) return NAN;"),
    ("e4m3_ties_odd", "if (dd < bestd || (dd == bestd && (c & 1u) == 0u)) {",
     "if (dd < bestd || (dd == bestd && (c & 1u) == 1u)) {"),
    ("e4m3_sign_dropped", "return best | sign;", "return best;"),
    ("fp8_wrong_max", "float s32 = amax / 448.0f;", "float s32 = amax / 240.0f;"),
    ("fp8_dequant_drops_scale", "What[rr * d + i] = sc * val * (Dr ? Dr[i] : 1.0);",
     "What[rr * d + i] = val * (Dr ? Dr[i] : 1.0);"),
    ("lowrank_A_transposed", "for (int64_t i = 0; i < d; ++i) acc += A[k * d + i] * X[t * d + i];",
     "for (int64_t i = 0; i < d; ++i) acc += A[(i % rank) * d + (k * d + i) / rank % d] * X[t * d + i];"),
]

RUNNER = r"""
import sys, traceback
sys.path[:0] = [{tests!r}, {oracle!r}]
import oracle_pins, ttq_oracle
O = ttq_oracle.Oracle({lib!r})
failed = []
for chk in oracle_pins.ALL_CHECKS:
    try:
        chk(O)
    except Exception:
        failed.append(chk.__name__)
print("FAILED:" + ",".join(failed))
sys.exit(1 if failed else 0)
"""


@pytest.fixture(scope="module")
def source():
    with open(ttq_oracle.SOURCE) as f:
        return f.read()


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_is_caught(source, name, old, new):
    assert source.count(old) == 1, f"mutant {name}: anchor text not found exactly once"
    lib = ttq_oracle.build_variant(source.replace(old, new))
    code = RUNNER.format(tests=HERE, oracle=os.path.dirname(ttq_oracle.SOURCE), lib=lib)
    proc = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=300)
    assert proc.returncode != 0, f"mutant {name} passed every pin:\n{proc.stdout}\n{proc.stderr}"
