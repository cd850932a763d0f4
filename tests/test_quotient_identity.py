"""The quotient identity the INT4/INT8 quantisers rely on, checked exhaustively on the CPU.

The quantisers form RN(w / s) for every weight without a division: with
r = RN(1/s) and q0 = RN(w * r), the residual e = w - q0 * s is exact (one fused
multiply-add) and RN(q0 + e * r) = RN(w / s) (Markstein's correction step,
"Computation of elementary functions on the IBM RISC System/6000 processor",
IBM J. Res. Dev. 34(1), 1990).  The scales are bf16 values, so their
significands take only 128 values; away from over- and underflow the identity
depends only on the significands.  This test compiles a small C program that
checks every bf16 significand of s against every binary32 significand of w, at
both relative exponents (quotient below and above 1): 2^31 cases, compared bit
for bit with the binary64 quotient rounded to binary32 (correctly rounded: 53
bits exceed twice 24 plus 2).  The CUDA quantisers' bit-exact parity with the
oracle (GPU tests) then covers the kernels themselves.
"""
import os
import shutil
import subprocess
import tempfile

import pytest

CHECK_C = r"""
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>
static float from_bits(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t to_bits(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }
int main(void)
{
    long bad = 0, total = 0;
    for (uint32_t sm = 0; sm < 128; ++sm) {
        const float s = from_bits((127u << 23) | (sm << 16));
        const float r = (float)(1.0 / (double)s);
        for (uint32_t we = 0; we < 2; ++we)
            for (uint32_t wm = 0; wm < (1u << 23); ++wm) {
                const float w = from_bits(((127u - we) << 23) | wm);
                const float want = (float)((double)w / (double)s);
                const float q0 = w * r;
                const float e = fmaf(-q0, s, w);
                const float q1 = fmaf(e, r, q0);
                ++total;
                if (to_bits(q1) != to_bits(want)) ++bad;
            }
    }
    printf("%ld %ld\n", total, bad);
    return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_reciprocal_quotient_is_correctly_rounded_for_every_bf16_scale():
    with tempfile.TemporaryDirectory() as d:
        src, exe = os.path.join(d, "q.c"), os.path.join(d, "q")
        open(src, "w").write(CHECK_C)
        subprocess.run(["gcc", "-O2", "-ffp-contract=off", "-o", exe, src, "-lm"], check=True)
        total, bad = map(int, subprocess.run([exe], check=True, capture_output=True, text=True).stdout.split())
    assert total == 2 * 128 * (1 << 23)
    assert bad == 0
