"""The NVFP4 residual r = fp32(x - code * sc) is computed with one fused
multiply-add, fma(code, -sc, x) (precision_attention_video_b200/csrc/ta_prep.cu,
nvfp4_residual; ta_attn_common.cuh, nvfp4_residual32, two lanes at a time with
fma.rn.f32x2).  The two agree because code * sc is exact in fp32: an e2m1
value has at most 2 significant bits, a ue4m3 scale at most 4, and their
product lies in [2^-10, 2688].  This checks it in C with the host's correctly
rounded fmaf: every e2m1 code (both signs) times every finite ue4m3 scale,
against a spread of x (random magnitudes, x near the product, signed zeros,
subnormals), comparing bit patterns so that the sign of a zero result counts
too.  A zero scale (the group of an all-zero block) is included."""

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
static const float E2M1[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};
static float ue4m3(unsigned c) {               /* c in 0 .. 0x7E */
  if (c < 8) return ldexpf((float)c, -9);      /* subnormals c * 2^-9 */
  return ldexpf(1.0f + (float)(c & 7) / 8.0f, (int)(c >> 3) - 7);
}
static uint32_t bits(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }
static uint64_t s = 88172645463325252ull;
static uint32_t rnd(void) { s ^= s << 13; s ^= s >> 7; s ^= s << 17; return (uint32_t)s; }
int main(void) {
  unsigned long long n = 0, bad = 0, inexact = 0;
  for (unsigned c = 0; c <= 0x7E; ++c) {
    const float sc = ue4m3(c);
    for (int code = 0; code < 16; ++code) {
      const float v = (code & 8) ? -E2M1[code & 7] : E2M1[code & 7];
      const float prod = v * sc;
      if ((double)prod != (double)v * (double)sc) ++inexact;
      float xs[64];
      int k = 0;
      xs[k++] = 0.0f; xs[k++] = -0.0f; xs[k++] = prod; xs[k++] = -prod;
      xs[k++] = nextafterf(prod, INFINITY); xs[k++] = nextafterf(prod, -INFINITY);
      xs[k++] = 0x1p-149f; xs[k++] = -0x1p-149f; xs[k++] = 0x1p-126f; xs[k++] = 3.0e38f;
      while (k < 64) {
        const uint32_t r = rnd();
        const float m = 1.0f + (float)(r & 0xFFFFF) / 1048576.0f;
        const int e = (int)((r >> 20) % 60) - 40;                /* 2^-40 .. 2^19 */
        xs[k++] = ((r >> 31) ? -1.0f : 1.0f) * ldexpf(m, e);
      }
      for (int i = 0; i < k; ++i) {
        const float x = xs[i];
        const float a = fmaf(v, -sc, x);
        const float b = x - prod;
        ++n;
        if (bits(a) != bits(b)) ++bad;
      }
    }
  }
  printf("%llu %llu %llu\n", n, bad, inexact);
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_residual_fma_equals_subtraction_of_the_exact_product():
    with tempfile.TemporaryDirectory() as d:
        src = os.path.join(d, "resid.c")
        exe = os.path.join(d, "resid")
        with open(src, "w") as f:
            f.write(C_SRC)
        subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-o", exe, src, "-lm"])
        out = subprocess.check_output([exe], timeout=120).decode().split()
    n, bad, inexact = (int(x) for x in out)
    assert n == 127 * 16 * 64
    assert inexact == 0
    assert bad == 0
