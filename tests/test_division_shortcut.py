"""The quantisers' scale division s32 = span / (2^b - 1) (and max|x| / 448 for
FP8 codes) must be the correctly rounded binary32 quotient: the oracle
divides, and the codes are compared bit for bit.  The kernels form it as
q0 = RN(x * r) with r = RN(1 / b), then one fused multiply-add correction
q = RN(q0 + RN(x - q0 b) r) (x - q0 b is exact), keeping q0 when the
correction is NaN (x infinite or NaN).

This test states that formula again in C and checks it against C's own
binary32 division (IEEE, correctly rounded) on every subnormal input, a
stride through all other non-negative finite inputs, the specials and the
neighbours of every power of two.  For 448 the comparison is on what the
quantiser keeps: the quotient floored at 2^-14, with everything above 65504
equal (binary16 round-up gives inf).  The full sweep over all 2^31 inputs
was run once at design time with no mismatch for 1, 3, 7, 15 (exact) and
448 (after the floor); this sample keeps that claim checked in the suite."""
from __future__ import annotations

import pathlib
import shutil
import subprocess

import pytest

SOURCE = r"""
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>
static float f_of(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t u_of(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }
static float floor14(float v) {
  if (!(v >= 6.103515625e-05f)) v = 6.103515625e-05f;
  if (v > 65504.0f) v = INFINITY;
  return v;
}
static float shortcut(float x, float b, float r) {
  const float q0 = x * r;
  const float e = fmaf(-q0, b, x);
  return e == e ? fmaf(e, r, q0) : q0;
}
static uint64_t checked, bad;
static void check(uint32_t bits, float b, float r, int floored) {
  const float x = f_of(bits);
  float want = x / b, got = shortcut(x, b, r);
  if (floored) { want = floor14(want); got = floor14(got); }
  ++checked;
  if (!(u_of(want) == u_of(got) || (want != want && got != got))) {
    if (bad < 5) printf("mismatch b=%g x=%a want=%a got=%a\n", b, x, want, got);
    ++bad;
  }
}
int main(void) {
  const float bs[] = {3.0f, 7.0f, 15.0f, 448.0f};
  const float rs[] = {0x1.555556p-2f, 0x1.24924ap-3f, 0x1.111112p-4f, 0x1.24924ap-9f};
  for (int k = 0; k < 4; ++k) {
    volatile float one = 1.0f;
    if (rs[k] != one / bs[k]) { printf("reciprocal constant %d is not RN(1/b)\n", k); return 2; }
    const int floored = bs[k] == 448.0f;
    for (uint32_t u = 0; u < 0x00800000u; ++u) check(u, bs[k], rs[k], floored);        /* subnormals */
    for (uint64_t u = 0x00800000u; u < 0x7f800000u; u += 13) check((uint32_t)u, bs[k], rs[k], floored);
    for (uint32_t e = 1; e < 255; ++e)                                                 /* around 2^k */
      for (int d = -3; d <= 3; ++d) check((e << 23) + (uint32_t)d, bs[k], rs[k], floored);
    check(0x7f7fffffu, bs[k], rs[k], floored);                                         /* FLT_MAX */
    check(0x7f800000u, bs[k], rs[k], floored);                                         /* inf */
    check(0x7fc00000u, bs[k], rs[k], floored);                                         /* NaN */
  }
  printf("checked %llu mismatches %llu\n", (unsigned long long)checked, (unsigned long long)bad);
  return bad != 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_constant_division_shortcut_is_correctly_rounded(tmp_path: pathlib.Path):
    src = tmp_path / "divsc.c"
    exe = tmp_path / "divsc"
    src.write_text(SOURCE)
    # no contraction: every operation rounds exactly as written (fmaf is the
    # fused one)
    subprocess.run(["gcc", "-O2", "-ffp-contract=off", "-o", str(exe), str(src), "-lm"], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stdout + out.stderr
    assert "mismatches 0" in out.stdout
