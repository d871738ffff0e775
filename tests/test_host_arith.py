"""Host-side checks of arithmetic identities the CUDA kernels rely on.

The quantisers compute the per-row step fl32(absmax / 127) with two fused
multiply-adds instead of a division (q0 = fl32(a c), c = fl32(1/127);
r = fma(-q0, 127, a); q = fma(r, c, q0)).  This test compiles a small C
program that compares that sequence with the IEEE quotient on a strided sweep
of every binary32 exponent (the kernels' comment records the exhaustive
sweep).  C's fmaf is the correctly rounded fused multiply-add, as the GPU's
is, and -ffp-contract=off keeps the other operations separate."""
import os
import shutil
import subprocess
import textwrap

import pytest

SRC = textwrap.dedent(r"""
    #include <math.h>
    #include <stdint.h>
    #include <stdio.h>
    #include <string.h>
    static float asf(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
    int main(void) {
      const float c = 1.0f / 127.0f;
      long long bad = 0, n = 0;
      for (uint32_t u = 0; u < 0x7f800000u; u += 61u) {  /* every exponent, strided mantissas */
        const float a = asf(u);
        volatile float ref = a / 127.0f;
        const float q0 = a * c;
        const float r = fmaf(-q0, 127.0f, a);
        const float q = fmaf(r, c, q0);
        bad += (q != ref);
        ++n;
      }
      for (uint32_t u = 0; u < 0x00800000u; ++u) {  /* all subnormals */
        const float a = asf(u);
        volatile float ref = a / 127.0f;
        const float q0 = a * c;
        const float q = fmaf(fmaf(-q0, 127.0f, a), c, q0);
        bad += (q != ref);
        ++n;
      }
      printf("%lld %lld\n", n, bad);
      return 0;
    }
""")


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_div127_fma_sequence(tmp_path):
    src = tmp_path / "div127.c"
    exe = tmp_path / "div127"
    src.write_text(SRC)
    subprocess.run(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-o", str(exe), str(src),
                    "-lm"], check=True)
    n, bad = map(int, subprocess.run([str(exe)], check=True, capture_output=True,
                                     text=True).stdout.split())
    assert n > 40_000_000 and bad == 0
