"""The activation kernel computes amax / 6 (NVFP4) and amax / 7 (INT4) with
the FMA division by a known constant of Markstein and of Brisebarre & Muller
("Accelerating correctly rounded floating-point division when the divisor is
known in advance", IEEE Trans. Computers, 2004):

    q0 = x * RN(1/d);  r = fma(-d, q0, x);  q = fma(r, RN(1/d), q0)

instead of an IEEE division.  Scaling x by a power of two scales q0, r and q
exactly while every value stays normal, so checking every significand of a
few binades checks every normal x.  This test runs that check in C (IEEE fp32,
fmaf, no contraction) and pins where the method equals x / d: everywhere for
d = 7, and for d = 6 from x = 2^-125 up (smaller x give subnormal quotients,
which round to the E4M3 scale 0 either way).
"""
import os
import subprocess
import tempfile

import pytest

C_SRC = r"""
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>
static float asf(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
int main(void) {
  const float ds[2] = {6.0f, 7.0f};
  const int exps[5] = {-125, -10, 0, 1, 126};
  for (int t = 0; t < 2; ++t) {
    volatile float d = ds[t];
    const float c = 1.0f / d;
    long bad = 0;
    for (int ei = 0; ei < 5; ++ei) {
      const uint32_t e = (uint32_t)(exps[ei] + 127);
      for (uint32_t m = 0; m < (1u << 23); ++m) {
        const float x = asf((e << 23) | m);
        const float q0 = x * c;
        const float r = fmaf(-d, q0, x);
        const float q = fmaf(r, c, q0);
        if (q != x / d) ++bad;
      }
    }
    long sub = 0;   /* the binade just below: subnormal quotients */
    for (uint32_t m = 0; m < (1u << 23); ++m) {
      const float x = asf((1u << 23) | m);
      const float q0 = x * c;
      const float r = fmaf(-d, q0, x);
      const float q = fmaf(r, c, q0);
      if (q != x / d) ++sub;
      if (q > 1e-30f || x / d > 1e-30f) { printf("unexpected magnitude\n"); return 2; }
    }
    printf("%g %ld %ld\n", (double)d, bad, sub);
  }
  return 0;
}
"""


@pytest.fixture(scope="module")
def results():
    with tempfile.TemporaryDirectory() as tmp:
        src = os.path.join(tmp, "d.c")
        exe = os.path.join(tmp, "d")
        with open(src, "w") as f:
            f.write(C_SRC)
        subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-o", exe, src, "-lm"])
        out = subprocess.check_output([exe], text=True)
    res = {}
    for line in out.strip().splitlines():
        d, bad, sub = line.split()
        res[float(d)] = (int(bad), int(sub))
    return res


def test_division_by_7_is_correctly_rounded(results):
    assert results[7.0] == (0, 0)


def test_division_by_6_is_correctly_rounded_above_2_to_minus_125(results):
    bad, sub = results[6.0]
    assert bad == 0
    # below 2^-125 the two quotients may differ, but both are < 1e-30: E4M3 scale 0
    assert sub >= 0
