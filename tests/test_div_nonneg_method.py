"""The tile kernels split a tile index into (row tile, column tile) with
floor(a / b) computed as trunc(RZ(a * RZ(1 / b))) plus one correction step
for a < 2^22.  This test runs the same binary32 operations on the host under
round-toward-zero for every b in 1..4096 against edge and random dividends
and compares with integer division."""
import ctypes
import os
import subprocess
import tempfile

SRC = r"""
#include <fenv.h>
#include <stdint.h>
#pragma STDC FENV_ACCESS ON
static int est(int a, int b) {
    volatile float fb = (float)b, fa = (float)a;
    fesetround(FE_TOWARDZERO);
    volatile float r = 1.0f / fb;
    volatile float p = fa * r;
    fesetround(FE_TONEAREST);
    int q = (int)p;
    if ((q + 1) * b <= a) ++q;
    return q;
}
int check(int *bad_a, int *bad_b) {
    uint32_t s = 12345u;
    for (int b = 1; b <= 4096; ++b) {
        int edges[8] = {0, 1, b - 1, b, b + 1, (1 << 22) - 1, ((1 << 22) - 1) / b * b, ((1 << 22) - 1) / b * b - 1};
        for (int i = 0; i < 8; ++i) {
            int a = edges[i];
            if (a < 0 || a >= (1 << 22)) continue;
            if (est(a, b) != a / b) { *bad_a = a; *bad_b = b; return 1; }
        }
        for (int k = 0; k < 512; ++k) {
            s = s * 1664525u + 1013904223u;
            int a = (int)(s >> 10);                       /* 0 .. 2^22 - 1 */
            if (est(a, b) != a / b) { *bad_a = a; *bad_b = b; return 1; }
            int m = a / b * b;                            /* exact multiples and their neighbours */
            if (est(m, b) != m / b || (m > 0 && est(m - 1, b) != (m - 1) / b)) { *bad_a = m; *bad_b = b; return 1; }
        }
    }
    return 0;
}
"""


def test_fast_tile_division_matches_integer_division():
    d = tempfile.mkdtemp(prefix="qz_divnn_")
    c = os.path.join(d, "divnn.c")
    so = os.path.join(d, "divnn.so")
    with open(c, "w") as fh:
        fh.write(SRC)
    subprocess.run(["gcc", "-O1", "-frounding-math", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC",
                    "-o", so, c, "-lm"], check=True)
    lib = ctypes.CDLL(so)
    a, b = ctypes.c_int(0), ctypes.c_int(0)
    assert lib.check(ctypes.byref(a), ctypes.byref(b)) == 0, (a.value, b.value)
