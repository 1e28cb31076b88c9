"""The NVFP4 block scale divides amax by 6 with one product and one FMA
correction (precision_attention_video_b200/csrc/ta_attn_common.cuh, div6)
instead of an IEEE division.  This checks, in C with the host's correctly
rounded fmaf, that the sequence returns the correctly rounded fp32 quotient
for inputs >= 2^-125 (every mantissa of the exponents where P' maxima lie, a
stride through all others; the whole float range was checked once the same
way), and that below 2^-125 it never changes the e4m3
code of the quotient (both round to 0 there)."""

import os
import shutil
import subprocess
import tempfile

import pytest

C_SRC = r"""
#include <stdio.h>
#include <math.h>
#include <stdint.h>
#include <string.h>
static float div6(float a) {
  const float r = 1.0f / 6.0f;
  const float q0 = a * r;
  return fmaf(fmaf(-6.0f, q0, a), r, q0);
}
int main(void) {
  unsigned long long n = 0, bad = 0, tiny_bad = 0;
  for (uint32_t u = 1; u < 0x7F800000u; ) {
    float a; memcpy(&a, &u, 4);
    const float ref = (float)((double)a / 6.0);   /* exact quotient, one rounding */
    const float q = div6(a);
    ++n;
    if (q != ref) {
      if (a >= 0x1p-125f) ++bad;
      else if (fabsf(ref) >= 0x1p-10f || fabsf(q) >= 0x1p-10f) ++tiny_bad;
    }
    const uint32_t e = u >> 23;
    /* every mantissa for exponents 2^-30 .. 2^16 (where P' maxima lie), a
       stride through all other exponents */
    u += (e >= 97u && e <= 143u) ? 1u : 4099u;
  }
  printf("%llu %llu %llu\n", n, bad, tiny_bad);
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_div6_matches_correctly_rounded_quotient():
    with tempfile.TemporaryDirectory() as d:
        src = os.path.join(d, "div6.c")
        exe = os.path.join(d, "div6")
        with open(src, "w") as f:
            f.write(C_SRC)
        subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-o", exe, src, "-lm"])
        out = subprocess.check_output([exe], timeout=300).decode().split()
    n, bad, tiny_bad = (int(x) for x in out)
    assert n > 300_000_000
    assert bad == 0
    assert tiny_bad == 0
