"""The quantizers' block-scale quotient RN(b / t) is computed without a
division instruction: y = RN(1 / t), q0 = RN(b * y), e = b - q0 * t (one
FMA, exact), q1 = RN(q0 + e * y) (one FMA) -- Markstein's FMA correction of a
reciprocal product.  The kernels use it for t >= 2^-60 and IEEE division
below.  This test checks, on the CPU, that q1 is the correctly rounded
quotient (bit for bit against IEEE binary32 division).

Why significands suffice: for t >= 2^-60 and quotients b / t in [2^-11,
2^10] -- every quotient that can reach a nonzero E4M3 code or its
saturation, since b <= amax = 2688 s_global and t = RN(6 s_global) -- y, q0, e
and q1 are normal binary32 numbers, so multiplying b or t by a power of two
scales every step exactly and leaves the comparison unchanged.  The check
therefore takes b and t in [1, 2): all 2^23 significands of b, exhaustively,
for each divisor significand of a set of 1024 (the structured ones 1, 1 +
2^-23, 2 - 2^-23, 1.5 and a seeded random sample)."""
import os
import shutil
import subprocess

import pytest

PROGRAM = r"""
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>
static float f_of(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t u_of(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }
int main(int argc, char** argv) {
    const int nd = atoi(argv[1]);
    uint64_t s = 0x9E3779B97F4A7C15ull;            /* xorshift64: the divisor sample */
    long long bad = 0, checks = 0;
    for (int d = 0; d < nd; ++d) {
        uint32_t mt;
        if (d == 0) mt = 0;
        else if (d == 1) mt = 1;
        else if (d == 2) mt = 0x7FFFFF;
        else if (d == 3) mt = 0x400000;
        else { s ^= s << 13; s ^= s >> 7; s ^= s << 17; mt = (uint32_t)(s >> 20) & 0x7FFFFF; }
        const float t = f_of(0x3F800000u | mt);
        const float y = 1.0f / t;                      /* RN(1 / t) */
        for (uint32_t mb = 0; mb < (1u << 23); ++mb) {
            const float b = f_of(0x3F800000u | mb);
            const float q0 = b * y;                    /* RN(b * y) */
            const float e = fmaf(-q0, t, b);           /* b - q0 t, exact */
            const float q1 = fmaf(e, y, q0);           /* RN(q0 + e y) */
            if (u_of(q1) != u_of(b / t)) {
                if (bad < 5) printf("mismatch t=%a b=%a q1=%a ref=%a\n", t, b, q1, b / t);
                ++bad;
            }
        }
        checks += 1 << 23;
    }
    printf("%lld %lld\n", checks, bad);
    return 0;
}
"""


def _has_hw_fma() -> bool:
    try:
        with open("/proc/cpuinfo") as f:
            return " fma " in f.read()
    except OSError:
        return False


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs a C compiler")
def test_fma_corrected_quotient_equals_ieee_division(tmp_path):
    src = tmp_path / "div.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "div"
    flags = ["-O3", "-std=c11", "-ffp-contract=off", "-fno-fast-math"]
    hw = _has_hw_fma()
    if hw:
        flags.append("-mfma")      # hardware fmaf; glibc's software fmaf is also correctly rounded, only slower
    subprocess.check_call(["gcc", *flags, str(src), "-o", str(exe), "-lm"])
    n_div = 1024 if hw else 128
    out = subprocess.run([str(exe), str(n_div)], capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr
    checks, bad = (int(v) for v in out.stdout.strip().splitlines()[-1].split())
    assert checks == n_div * (1 << 23)
    assert bad == 0, out.stdout
