"""The pack kernel's group scale m / 6 is formed without a division: the
product by c = RN(1/6) corrected once by two fmas (Markstein's correction, as
used for division by a constant known in advance by Brisebarre, Muller and
Raina, 2004), with a real division below m = 2^-122 where quotients are
subnormal.  This checks that scheme, written out in C with the C library's
correctly rounded fmaf, against IEEE division of fp32 values: every m in the
binades where intermediate residuals can be subnormal ([2^-122, 2^-100)), the
binade [1, 2) (the scheme is invariant under scaling by powers of two once no
intermediate is subnormal), the top binade, and the exact threshold."""
import shutil
import subprocess

import pytest

SRC = r"""
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>
static float f(uint32_t u) { float x; memcpy(&x, &u, 4); return x; }
static float div6(float m) {
    if (m < 0x1p-122f) return m / 6.0f;
    const float c = 0x1.555556p-3f;
    const float q0 = m * c;
    const float r = fmaf(-q0, 6.0f, m);
    return fmaf(r, c, q0);
}
static unsigned long long check(uint32_t lo, uint32_t hi) {
    unsigned long long bad = 0;
    for (uint64_t u = lo; u < hi; ++u) {
        const float m = f((uint32_t)u), q = div6(m), ref = m / 6.0f;
        if (memcmp(&q, &ref, 4) != 0) ++bad;
    }
    return bad;
}
int main(void) {
    /* c is RN(1/6) */
    if (0x1.555556p-3f != 1.0f / 6.0f) { puts("constant"); return 2; }
    unsigned long long bad = 0;
    bad += check(0x00000000u, 0x00001000u);   /* zero and the smallest subnormals */
    bad += check(0x027FF000u, 0x06000000u);   /* 2^-122 (threshold) .. 2^-115 */
    bad += check(0x06000000u, 0x0D800000u);   /* .. 2^-100 */
    bad += check(0x3F800000u, 0x40000000u);   /* [1, 2) */
    bad += check(0x7F000000u, 0x7F800000u);   /* top binade up to FLT_MAX */
    printf("%llu\n", bad);
    return bad != 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_division_free_scale_is_correctly_rounded(tmp_path):
    src = tmp_path / "div6.c"
    src.write_text(SRC)
    exe = tmp_path / "div6"
    subprocess.run(["gcc", "-O2", "-ffp-contract=off", str(src), "-o", str(exe), "-lm"],
                   check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == "0", r.stdout + r.stderr
