"""The kernels compute RN(b / 6) for the NVFP4 block scale with one FMA
quotient correction instead of a full IEEE division.  This test runs the same
three IEEE operations (binary32 multiply, fma, fma; C's fmaf is correctly
rounded) on the host for every positive finite bf16 value b and compares with
the IEEE binary32 quotient b / 6.0f: the method is exact on the whole domain
the kernels feed it."""
import ctypes
import os
import subprocess
import tempfile

import numpy as np

SRC = r"""
#include <math.h>
#include <stdint.h>
#include <string.h>
static float f(uint32_t u) { float x; memcpy(&x, &u, 4); return x; }
static uint32_t u(float x) { uint32_t v; memcpy(&v, &x, 4); return v; }
int check(uint32_t *bad_out) {
    const float c = 1.0f / 6.0f;
    int bad = 0;
    for (uint32_t h = 1; h < 0x7F80u; ++h) {          /* every positive finite bf16 */
        float b = f(h << 16);
        float q0 = b * c;
        float r = fmaf(-q0, 6.0f, b);
        float q = fmaf(r, c, q0);
        if (u(q) != u(b / 6.0f)) { if (bad < 4) bad_out[bad] = h; ++bad; }
    }
    return bad;
}
"""


def test_div6_correction_is_exact_for_every_bf16():
    d = tempfile.mkdtemp(prefix="qz_div6_")
    c = os.path.join(d, "div6.c")
    so = os.path.join(d, "div6.so")
    with open(c, "w") as fh:
        fh.write(SRC)
    subprocess.run(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC", "-o", so, c, "-lm"],
                   check=True)
    lib = ctypes.CDLL(so)
    bad = (ctypes.c_uint32 * 4)()
    n = lib.check(bad)
    assert n == 0, [hex(b) for b in bad[: min(n, 4)]]
