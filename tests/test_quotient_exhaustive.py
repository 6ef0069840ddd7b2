"""The FP8 cache quantiser's quotient, checked exhaustively on the CPU.

The codes of an FP8 cache row are the e4m3 round-to-nearest-even of the float32 quotient
x / scale, scale = RN(max|x| / 448) (value = scale * code; "HySparse2: Hybrid Sparse Attention
with Two-Level KV Sharing", bullet "Inference cost": FP8 cache). The kernels form the quotient
with Markstein's correction of the reciprocal product (r = RN(1 / scale); q0 = RN(x r);
e = fma(-scale, q0, x); q = fma(e, r, q0)) for scales in [2^-100, 2^100], and divide directly
otherwise. This test runs that arithmetic, in C with the C library's correctly rounded fmaf,
over every pair of non-negative finite bf16 values x <= a (a = the row maximum), about 5.3e8
pairs, and requires:
  * the float32 value equal to the IEEE quotient x / scale whenever that is >= 2^-11
    (below it every value, exact or not, has the e4m3 code 0),
  * the e4m3 code equal to the code of the IEEE quotient, always.
Rounding to nearest is symmetric in the sign, so negative x behave as their magnitudes."""
import os
import subprocess

import pytest

SRC = r"""
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>
static float bf(uint32_t b) { uint32_t u = b << 16; float f; memcpy(&f, &u, 4); return f; }
/* e4m3fn round-to-nearest-even of a non-negative float32, saturating at 448 */
static int e4m3(float y) {
  double a = fabs((double)y);
  if (a > 448.0) a = 448.0;
  if (a < ldexp(1.0, -6)) return (int)rint(a / ldexp(1.0, -9));
  int e; frexp(a, &e); e -= 1;
  int q = (int)rint((a / ldexp(1.0, e) - 1.0) * 8.0), E = e + 7;
  if (q == 8) { q = 0; E += 1; }
  int code = (E << 3) | q;
  return code > 0x7e ? 0x7e : code;
}
int main(void) {
  long long pairs = 0, value_bad = 0, code_bad = 0;
  for (uint32_t ab = 1; ab < 0x7f80; ++ab) {
    const float a = bf(ab), s = a / 448.0f;
    const int fast = s >= 0x1p-100f && s <= 0x1p100f;
    const float r = 1.0f / s;
    for (uint32_t xb = 0; xb <= ab; ++xb) {
      const float x = bf(xb), q = x / s;
      float k;
      if (fast) {
        const float q0 = x * r;
        const float e = fmaf(-s, q0, x);
        k = fmaf(e, r, q0);
      } else {
        k = x / s;
      }
      ++pairs;
      if (q >= 0x1p-11f && k != q) ++value_bad;
      if (signbit(k) || e4m3(k) != e4m3(q)) ++code_bad;
    }
  }
  printf("%lld %lld %lld\n", pairs, value_bad, code_bad);
  return 0;
}
"""


def test_markstein_quotient_matches_ieee_division_on_every_bf16_pair(tmp_path):
    src = tmp_path / "quotient.c"
    exe = tmp_path / "quotient"
    src.write_text(SRC)
    subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-o", str(exe),
                           str(src), "-lm"])
    pairs, value_bad, code_bad = map(int, subprocess.check_output([str(exe)], timeout=600).split())
    assert pairs > 5 * 10 ** 8
    assert value_bad == 0
    assert code_bad == 0
