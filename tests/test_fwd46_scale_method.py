"""The forward quantizer's group scale without a division per group.

The scale of a candidate grid k is RNE_E4M3(RN(a / (g k))).  The kernels form t' = RN(a *
RN(1/(g k))) instead and keep it when it lies in the E4M3 normal range (t' >= 2^-6) with its 20
bits below the E4M3 mantissa more than 3 ulps from the rounding midpoint 0x80000; otherwise they
form the quotient itself.  Why this is exact: t' and RN(a/(g k)) differ by at most 3 ulps (two
roundings of relative size at most 2^-24 each, against an ulp of at least 2^-24 of the value),
so when no E4M3 rounding boundary lies within 3 ulps of t', both round to the same E4M3 value.
These CPU checks emulate the kernels' binary32 steps with numpy (IEEE round-to-nearest-even)
and compare with the exact definition over every significand of several binades, random values
across the whole range, and values placed right at the E4M3 midpoints."""
import ml_dtypes
import numpy as np

F32 = np.float32


def e4m3_rne(t: np.ndarray) -> np.ndarray:
    """RNE onto E4M3 with saturation at 448 (the library's and the oracle's rule)."""
    return np.minimum(t, F32(448.0)).astype(ml_dtypes.float8_e4m3fn).view(np.uint8)


def fast(a: np.ndarray, gk: np.float32):
    inv = F32(1.0) / gk
    tp = (a * inv).astype(F32)
    low = tp.view(np.uint32) & np.uint32(0xFFFFF)
    safe = (tp >= F32(2.0 ** -6)) & ((low < 0x80000 - 3) | (low > 0x80000 + 3))
    exact = (a / gk).astype(F32)
    return np.where(safe, e4m3_rne(tp), e4m3_rne(exact)), safe, tp, exact


def _check(a: np.ndarray, gk: np.float32):
    got, safe, tp, exact = fast(a, gk)
    want = e4m3_rne((a / gk).astype(F32))
    assert np.array_equal(got, want), np.argwhere(got != want)[:5]
    # the 3-ulp bound behind the shortcut
    ulp = np.spacing(exact)
    assert np.all(np.abs(tp.astype(np.float64) - exact.astype(np.float64)) <= 3 * ulp.astype(np.float64))
    return safe


def test_every_significand_of_several_binades():
    rng = np.random.default_rng(0)
    for _ in range(3):
        A = F32(rng.uniform(0.5, 40.0))
        g = F32(A / F32(1792.0))
        for k in (6.0, 4.0):
            gk = F32(g * F32(k))
            for e in (-3, 2, 8):                       # t from about 2^-5 to 2^10
                base = np.uint32((127 + e) << 23)
                a = (np.arange(1 << 23, dtype=np.uint32) + base).view(F32)
                a = a * gk                              # a spans the binade's t range times gk
                safe = _check(a.astype(F32), gk)
                assert safe.mean() > 0.99


def test_random_values_across_the_range_and_tiny_groups():
    rng = np.random.default_rng(1)
    for _ in range(8):
        A = F32(10.0 ** rng.uniform(-30, 30))
        g = F32(A / F32(1792.0))
        for k in (6.0, 4.0):
            gk = F32(g * F32(k))
            a = (F32(A) * rng.uniform(0, 1, 1 << 20) ** 8).astype(F32)   # many groups far below A
            a[:16] = 0.0
            _check(a, gk)


def test_values_at_the_e4m3_midpoints_take_the_exact_path():
    g = F32(3.7 / 1792.0)
    gk = F32(g * F32(6.0))
    vals = np.array([ml_dtypes.float8_e4m3fn(v) for v in np.arange(1, 126, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn)],
                    dtype=np.float64)
    mids = (vals[:-1] + vals[1:]) / 2
    mids = mids[mids >= 2.0 ** -6]
    t = mids.astype(F32)
    off = np.arange(-6, 7, dtype=np.int64)
    tb = (t.view(np.uint32)[:, None].astype(np.int64) + off[None, :]).astype(np.uint32).view(F32).ravel()
    a = (tb * gk).astype(F32)
    safe = _check(a, gk)
    assert (~safe).sum() > 0
