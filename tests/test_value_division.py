"""The value encoder computes the scale (max - min) / L, L = 2^b - 1, without a division instruction:
q = RN(x * RN(1/L)), then one FMA correction with the exact residual fma(-q, L, x).  This checks that formula
against IEEE division on the host (hardware FMA, gcc) for non-negative finite fp32 x: every 61st bit pattern
by default (all exponents, subnormals included), every pattern with TQ_EXHAUSTIVE=1 (about 1.5 min)."""
import os
import shutil
import subprocess
import tempfile

import pytest

_SRC = r"""
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>
int main(int argc, char** argv) {
    const uint64_t stride = strtoull(argv[1], 0, 10);
    const float Ls[4] = {3.f, 7.f, 15.f, 255.f};
    unsigned long long bad = 0, n = 0;
    for (int li = 0; li < 4; ++li) {
        const float L = Ls[li], y = 1.0f / L;
        for (uint64_t u = 0; u < 0x7F800000ull; u += stride) {
            float x;
            uint32_t w = (uint32_t)u;
            memcpy(&x, &w, 4);
            const float q = x * y;
            const float q2 = fmaf(fmaf(-q, L, x), y, q);
            bad += (q2 != x / L);
            ++n;
        }
    }
    printf("%llu %llu\n", bad, n);
    return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_fma_corrected_division_by_level_count():
    stride = 1 if os.environ.get("TQ_EXHAUSTIVE") == "1" else 61
    with tempfile.TemporaryDirectory() as tmp:
        src, exe = os.path.join(tmp, "div.c"), os.path.join(tmp, "div")
        with open(src, "w") as f:
            f.write(_SRC)
        # -mfma: fmaf is the single-rounding hardware FMA; -ffp-contract=off: no other fusion
        subprocess.run(["gcc", "-O2", "-mfma", "-ffp-contract=off", src, "-o", exe, "-lm"], check=True)
        out = subprocess.run([exe, str(stride)], check=True, capture_output=True, text=True).stdout.split()
    bad, n = int(out[0]), int(out[1])
    assert n > 4 * (0x7F800000 // stride) - 8
    assert bad == 0
