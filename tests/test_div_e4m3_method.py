"""The kernels compute the NVFP4 element multiplier RN(S / s), s an e4m3
block scale m * 2^k (m = 1..15), as RN(S / m) * 2^-k with one FMA quotient
correction (q0 = RN(S * c), c = RN(1/m); r = S - m q0 exactly; q =
RN(q0 + r c)) -- Markstein's correction, exact when c is the correctly
rounded reciprocal and m has few significant bits.  Rounding of S / m depends
only on the significand of S, so running every binary32 significand (one
binade) for every m = 1..15 is an exhaustive check of the method against IEEE
division."""
import ctypes
import os
import subprocess
import tempfile

SRC = r"""
#include <math.h>
#include <stdint.h>
#include <string.h>
static float f(uint32_t u) { float x; memcpy(&x, &u, 4); return x; }
static uint32_t u(float x) { uint32_t v; memcpy(&v, &x, 4); return v; }
long check(uint32_t *bad_out) {
    long bad = 0;
    for (int m = 1; m <= 15; ++m) {
        const float fm = (float)m;
        const float c = 1.0f / fm;
        for (uint32_t mant = 0; mant < (1u << 23); ++mant) {
            float S = f((127u << 23) | mant);          /* [1, 2) */
            float q0 = S * c;
            float r = fmaf(-q0, fm, S);
            float q = fmaf(r, c, q0);
            if (u(q) != u(S / fm)) { if (bad < 4) bad_out[bad] = (uint32_t)(m << 24) | mant; ++bad; }
        }
    }
    return bad;
}
"""


def test_div_by_e4m3_significand_is_exact():
    d = tempfile.mkdtemp(prefix="qz_dive4m3_")
    c = os.path.join(d, "dive4m3.c")
    so = os.path.join(d, "dive4m3.so")
    with open(c, "w") as fh:
        fh.write(SRC)
    subprocess.run(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC", "-o", so, c, "-lm"],
                   check=True)
    lib = ctypes.CDLL(so)
    lib.check.restype = ctypes.c_long
    bad = (ctypes.c_uint32 * 4)()
    n = lib.check(bad)
    assert n == 0, (n, [hex(b) for b in bad[: min(n, 4)]])
