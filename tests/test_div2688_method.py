"""The row-scaled NVFP4 kernel computes the decode scale RN(A / 2688) of a
row amax A with one FMA quotient correction instead of a full IEEE division.
This test runs the same three IEEE operations (binary32 multiply, fma, fma;
C's fmaf is correctly rounded) on the host for every bf16 value A from 2^-100
(the smallest amax the NVFP4 contract admits) to the largest finite one, and
compares with the IEEE binary32 quotient A / 2688.0f, then with the encode
scale RN(1 / g) taken from it."""
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
int check(uint32_t lo, uint32_t *bad_out, int *count) {
    const float c = 1.0f / 2688.0f;
    int bad = 0, n = 0;
    for (uint32_t h = lo; h < 0x7F80u; ++h) {         /* bf16 bit patterns from lo to the largest finite */
        float A = f(h << 16);
        float q0 = A * c;
        float r = fmaf(-q0, 2688.0f, A);
        float g = fmaf(r, c, q0);
        float ref = A / 2688.0f;
        ++n;
        if (u(g) != u(ref) || u(1.0f / g) != u(1.0f / ref)) { if (bad < 4) bad_out[bad] = h; ++bad; }
    }
    *count = n;
    return bad;
}
"""


def test_div2688_correction_is_exact_on_the_contract_domain():
    d = tempfile.mkdtemp(prefix="qz_div2688_")
    c = os.path.join(d, "div2688.c")
    so = os.path.join(d, "div2688.so")
    with open(c, "w") as fh:
        fh.write(SRC)
    subprocess.run(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC", "-o", so, c, "-lm"],
                   check=True)
    lib = ctypes.CDLL(so)
    bad = (ctypes.c_uint32 * 4)()
    count = ctypes.c_int(0)
    lo = (127 - 100) << 7  # bf16 bits of 2^-100
    n = lib.check(lo, bad, ctypes.byref(count))
    assert count.value == 0x7F80 - lo
    assert n == 0, [hex(b) for b in bad[: min(n, 4)]]


def test_plain_reciprocal_product_is_not_exact():
    """Without the correction step, RN(A * RN(1/2688)) differs from the IEEE
    quotient for some bf16 A in the same domain, so the check above
    discriminates."""
    src = SRC.replace("float g = fmaf(r, c, q0);", "float g = q0; (void)r;")
    d = tempfile.mkdtemp(prefix="qz_div2688n_")
    c = os.path.join(d, "div2688n.c")
    so = os.path.join(d, "div2688n.so")
    with open(c, "w") as fh:
        fh.write(src)
    subprocess.run(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC", "-o", so, c, "-lm"],
                   check=True)
    lib = ctypes.CDLL(so)
    bad = (ctypes.c_uint32 * 4)()
    count = ctypes.c_int(0)
    assert lib.check((127 - 100) << 7, bad, ctypes.byref(count)) > 0
