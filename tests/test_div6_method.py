"""Host check of the MS-EDEN producer's division by 6 (no GPU needed).

The kernel computes the group scale p = a / 6 rounded to nearest-even as
q0 = RN(a * RN(1/6)), rem = fma(-q0, 6, a) (exact), p = fma(rem, RN(1/6), q0)
(Markstein's FMA correction step).  IEEE binary32 multiply and fused multiply-add give the same
bits on the host as on the GPU, so restating the three steps in C and comparing them with the
correctly rounded quotient over every significand of a binade proves the method: scaling a by a
power of two scales q0, rem and p exactly in [2^-100, 2^128), the range the kernel uses (groups
below 2^-100 are flushed before the division).  The two extreme binades are checked directly.
"""
import ctypes
import os
import subprocess
import tempfile

SRC = r"""
#include <math.h>
#include <stdint.h>
#include <string.h>
static float f32(uint32_t u) { float x; memcpy(&x, &u, 4); return x; }
static uint32_t bits(float x) { uint32_t v; memcpy(&v, &x, 4); return v; }
long mismatches(uint32_t biased_exponent) {
    const float sixth = 1.0f / 6.0f;
    long bad = 0;
    for (uint32_t m = 0; m < (1u << 23); ++m) {
        const float a = f32((biased_exponent << 23) | m);
        const float q0 = a * sixth;
        const float rem = fmaf(-q0, 6.0f, a);
        const float p = fmaf(rem, sixth, q0);
        /* a / 6 is never a binary32 tie unless exact, so the double quotient rounds once */
        const float ref = (float)((double)a / 6.0);
        bad += bits(p) != bits(ref);
    }
    return bad;
}
"""


def _lib():
    d = tempfile.mkdtemp(prefix="qt2_div6_")
    src, so = os.path.join(d, "div6.c"), os.path.join(d, "div6.so")
    with open(src, "w") as f:
        f.write(SRC)
    subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC", src, "-o", so,
                           "-lm"])
    lib = ctypes.CDLL(so)
    lib.mismatches.restype = ctypes.c_long
    lib.mismatches.argtypes = [ctypes.c_uint32]
    return lib


def test_div6_is_correctly_rounded():
    lib = _lib()
    for biased in (127, 127 - 100, 254):   # [1, 2), [2^-100, 2^-99), [2^127, 2^128)
        assert lib.mismatches(biased) == 0, biased
