"""Pins of the oracle's number formats and random stream (CPU only).

Each check compares the oracle with something other than itself: the grid the pages name,
library casts (ml_dtypes, torch float8) that implement IEEE round-to-nearest-even, the
defining property of round-to-nearest, the exact expectation of stochastic rounding, and
the published Philox known-answer vectors.
"""
import os

import ml_dtypes
import numpy as np
import pytest
import torch

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


# ----------------------------------------------------------------------------- E2M1
def test_e2m1_decode_is_the_nvfp4_grid():
    rows = _read_golden("e2m1_grid.txt")
    assert len(rows) == 8
    for code_s, mag_s in rows:
        code, mag = int(code_s), float(mag_s)
        assert O.e2m1_value(code) == mag
        neg = O.e2m1_value(code | 8)
        assert neg == -mag and (mag != 0.0 or np.signbit(neg))


def _e2m1_probe_values():
    mags = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    vals = []
    for a, b in zip(mags[:-1], mags[1:]):
        mid = np.float32((a + b) / 2)
        vals += [mid, np.nextafter(mid, np.float32(0)), np.nextafter(mid, np.float32(10))]
    vals += mags + [6.5, 7.0, 100.0, 1e30, np.inf, 1e-30, 1e-45, 0.1, 0.2499999]
    rng = np.random.default_rng(1)
    vals += list(rng.uniform(0, 8, 4000).astype(np.float32))
    vals += list(np.float32(2.0) ** rng.uniform(-30, 4, 1000).astype(np.float32))
    v = np.array(vals, dtype=np.float32)
    return np.concatenate([v, -v])


def test_e2m1_encode_matches_library_rne():
    v = _e2m1_probe_values()
    lib_codes = v.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    ours = np.array([O.e2m1_encode(float(x)) for x in v], dtype=np.uint8)
    finite = np.isfinite(v)
    assert np.array_equal(ours[finite], lib_codes[finite])
    # +-inf saturates to +-6 by our reading (satfinite)
    assert all(O.e2m1_encode(float(x)) == (7 if x > 0 else 15) for x in v[~finite])


def test_e2m1_encode_is_nearest_point():
    grid = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    for x in _e2m1_probe_values()[:3000]:
        if not np.isfinite(x):
            continue
        c = O.e2m1_encode(float(x))
        got = abs(O.e2m1_value(c))
        best = np.min(np.abs(abs(float(x)) - grid))
        assert abs(abs(float(x)) - got) == best
        # sign is kept, including for values that round to zero
        assert bool(c & 8) == bool(np.signbit(x))


# ----------------------------------------------------------------------------- E4M3
def test_e4m3_decode_matches_library():
    codes = np.arange(127, dtype=np.uint8)
    lib_vals = codes.view(ml_dtypes.float8_e4m3fn).astype(np.float32)
    ours = np.array([O.e4m3_value(int(c)) for c in codes], dtype=np.float32)
    assert np.array_equal(ours, lib_vals)
    assert O.e4m3_value(126) == 448.0 and O.e4m3_value(1) == 2.0 ** -9 and O.e4m3_value(8) == 2.0 ** -6


def test_e4m3_rne_matches_torch_cast():
    vals = [O.e4m3_value(c) for c in range(127)]
    probes = []
    for a, b in zip(vals[:-1], vals[1:]):
        m = np.float32((a + b) / 2)
        probes += [m, np.nextafter(m, np.float32(0)), np.nextafter(m, np.float32(1e9)), np.float32(a)]
    rng = np.random.default_rng(2)
    probes += list(np.float32(2.0) ** rng.uniform(-12, 8.8, 5000).astype(np.float32))
    p = np.array([x for x in probes if x <= 448.0], dtype=np.float32)
    ref = torch.from_numpy(p).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ours = np.array([O.e4m3_rne(float(x)) for x in p], dtype=np.uint8)
    assert np.array_equal(ours, ref)


def test_e4m3_rne_saturates_and_handles_zero():
    for v in [448.0, 449.0, 463.9, 464.0, 480.0, 1e6, float("inf")]:
        assert O.e4m3_rne(v) == 126
    assert O.e4m3_rne(0.0) == 0
    assert O.e4m3_rne(2.0 ** -10) == 0       # half the smallest subnormal: tie -> even (0)
    assert O.e4m3_rne(2.0 ** -10 * 1.0001) == 1


def _sr_count_up(v):
    """Number of the 2^20 draws u20 that round v up (monotone in u20: find it by bisection)."""
    lo_code = O.e4m3_sr(v, 0xFFFFFFFF)
    lo, hi = 0, 1 << 20     # first u20 that does not round up lies in [lo, hi]
    while lo < hi:
        mid = (lo + hi) // 2
        if O.e4m3_sr(v, mid << 12) != lo_code:
            lo = mid + 1
        else:
            hi = mid
    return lo, lo_code


def test_e4m3_sr_exact_expectation_bisection():
    rng = np.random.default_rng(3)
    vs = list(np.float32(2.0) ** rng.uniform(-6, 8.7, 300).astype(np.float32)) + [np.float32(2 ** -6), np.float32(1.0),
                                                                                  np.float32(447.9)]
    for v in vs:
        v = float(v)
        if v >= 448:
            continue
        count_up, lo_code = _sr_count_up(v)
        lo = O.e4m3_value(lo_code)
        if lo == v:
            assert count_up == 0
            continue
        hi = O.e4m3_value(lo_code + 1)
        assert lo < v < hi
        # E[result] = (count_up*hi + (2^20-count_up)*lo) / 2^20 must equal v exactly
        assert count_up * hi + ((1 << 20) - count_up) * lo == v * (1 << 20)


def test_e4m3_sr_full_enumeration():
    for v in [0.7890625 + 2 ** -20, 3.3333332538604736, 300.0001]:
        v = float(np.float32(v))
        u = np.arange(1 << 20, dtype=np.uint64) << np.uint64(12)
        f = O.lib().or_e4m3_sr
        res = np.fromiter((f(v, int(x)) for x in u[::64]), dtype=np.uint8, count=len(u[::64]))
        vals = np.array([O.e4m3_value(int(c)) for c in np.unique(res)])
        assert len(vals) <= 2 and vals.min() <= v <= vals.max()
        mean = np.mean([O.e4m3_value(int(c)) for c in res])
        assert abs(mean - v) <= (vals.max() - vals.min()) / 2 ** 13


# ----------------------------------------------------------------------------- Philox
def test_philox_known_answers():
    rows = _read_golden("philox4x32_10_kat.txt")
    assert len(rows) == 3
    for r in rows:
        vals = [int(x, 16) for x in r]
        ctr, key, out = vals[0:4], vals[4:6], vals[6:10]
        assert O.philox4x32_10(ctr, key) == out


def test_philox_word_indexing():
    seed = 0x0123456789ABCDEF
    for tid in (0, 3):
        for blk in (0, 1, 7, (1 << 32) + 5):
            block = O.philox4x32_10([blk & 0xFFFFFFFF, blk >> 32, tid, 0], [seed & 0xFFFFFFFF, seed >> 32])
            for w in range(4):
                assert O.philox_word(seed, tid, blk * 4 + w) == block[w]


def test_rht_signs_follow_word_bits():
    for seed in (0, 1, 12345):
        s = O.rht_signs(seed)
        words = O.philox4x32_10([0, 0, 0, 0], [seed & 0xFFFFFFFF, seed >> 32])
        for i in range(128):
            bit = (words[i >> 5] >> (i & 31)) & 1
            assert s[i] == (-1.0 if bit else 1.0)
        assert 30 < int((s < 0).sum()) < 98


def test_nonfinite_inputs_are_refused():
    """The quantizers are defined on finite values: inf or NaN anywhere in the input is refused
    (the library reports the same inputs as QT2_ERR_NONFINITE)."""
    import pytest
    import torch
    for bad in (float("inf"), float("-inf"), float("nan")):
        x = torch.zeros((128, 128), dtype=torch.bfloat16)
        x[5, 77] = bad
        for fn in (lambda t: O.fwd46(t), lambda t: O.msedEN(t, 1, 1, "row"), lambda t: O.msedEN(t, 1, 2, "col"),
                   lambda t: O.sr(t, 1, 1, "row"), lambda t: O.fwd46_sq(t), lambda t: O.fwd46_local(t)):
            with pytest.raises(ValueError):
                fn(x)
    # the largest finite bf16 is accepted
    x = torch.full((128, 128), 3.3895313892515355e38, dtype=torch.bfloat16)
    assert np.isfinite(O.fwd46(x).g)


def test_rotation_overflow_is_refused():
    """Finite inputs whose 128-point rotation overflows binary32 are refused by the rotating
    quantizers (the library reports them as QT2_ERR_NONFINITE); the forward quantizer, which
    does not rotate, takes them."""
    import pytest
    import torch
    x = torch.full((128, 128), 2.0 ** 125, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        O.msedEN(x, 1, 1, "row")
    with pytest.raises(ValueError):
        O.sr(x, 1, 1, "row")
    assert np.isfinite(O.fwd46(x).g)
