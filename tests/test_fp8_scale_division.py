"""The FP8 group scale RN(amax / 448) is formed without a division: with
c = RN(1/448), q0 = RN(amax * c), r = fma(-q0, 448, amax) (exact) and
q1 = fma(r, c, q0) (Markstein's division by a constant).  This checks, for
every non-negative finite fp32 amax, that q1 is the correctly rounded
quotient wherever that quotient is a normal number, and that every miss lies
below 2^-100 (where the kernels take the IEEE division instead).  The
reference is the fp64 quotient rounded to fp32: a/448 = a/(7 * 2^6) is either
exact in fp32 or has a binary expansion of period 3 past its leading bits, so
rounding it first to fp64 cannot land on an fp32 rounding midpoint."""
import os
import shutil
import subprocess

import pytest

SRC = r"""
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>
static float f_of(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
int main(void) {
    const float c = (float)(1.0 / 448.0);
    if (c != 0x1.24924ap-9f) { printf("constant %a\n", c); return 2; }
    unsigned long long bad_normal = 0, bad_fast = 0;
    #pragma omp parallel for reduction(+:bad_normal,bad_fast) schedule(static)
    for (long long i = 0; i < 0x7F800000LL; ++i) {
        const float a = f_of((uint32_t)i);
        const float q0 = a * c;
        const float r = fmaf(-q0, 448.0f, a);
        const float q1 = fmaf(r, c, q0);
        const float ref = (float)((double)a / 448.0);
        if (memcmp(&q1, &ref, 4) != 0) {
            if (ref >= 0x1p-126f) ++bad_normal;
            if (a >= 0x1p-100f) ++bad_fast;
        }
    }
    printf("%llu %llu\n", bad_normal, bad_fast);
    return 0;
}
"""


def test_group_scale_division_is_correctly_rounded(tmp_path):
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not available")
    src = tmp_path / "div448.c"
    src.write_text(SRC)
    exe = tmp_path / "div448"
    # strict IEEE fp32 evaluation: no contraction of a * c into an FMA, no
    # excess precision
    subprocess.run([gcc, "-O2", "-march=native", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-o", str(exe),
                    str(src), "-lm"], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True,
                         env={**os.environ, "OMP_NUM_THREADS": str(os.cpu_count() or 1)})
    bad_normal, bad_fast = map(int, out.stdout.split())
    assert bad_normal == 0
    assert bad_fast == 0
