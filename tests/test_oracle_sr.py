"""Pins of the oracle's binary32 elementwise-SR quantizer (the GPU SR baseline's contract; CPU).

Independent checks: every dequantized element is one of the two E2M1 grid neighbours of the
rotated value (scaled), and no element needs clipping (the group scale covers the group max);
the estimate is unbiased over 2048 seeds; it agrees with the fp64 SR baseline (already pinned
by its own unbiasedness test) on all but a handful of elements where binary32 and binary64
rounding of the same quantities differ; the MSE ratio to MS-EDEN holds the pages' "more than
2x lower error" claim at the same margin; zero and tiny groups.
"""
import numpy as np
import torch

import oracle as O
from tests.test_oracle_msedEN import _bf16, _bias_inputs, _mean_stats, _rotated, _unpack, strict_unbiased

GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _dequant_rotated(v: O.View) -> np.ndarray:
    return v.dequant()


def test_neighbours_and_no_clipping():
    rng = np.random.default_rng(3)
    xf = rng.standard_normal((8, 512)).astype(np.float32)
    xf[2, 7] = 40.0
    xf[5] *= 1e-3
    x = _bf16(xf)
    seed = 5
    v = O.sr(x, seed, 7, "row")
    y = _rotated(x, seed).astype(np.float64)
    R, C = y.shape
    s_val = np.array([O.e4m3_value(c) for c in range(256)], np.float64)[v.scales]
    d = np.repeat(s_val * np.float64(v.g), 16, axis=1)
    mag = np.abs(y) / d
    # the group scale covers the group: |y| / d <= 6 up to binary32 rounding of d and 1/d
    assert np.all(mag <= 6.0 * (1 + 2.0 ** -21))
    q = np.abs(v.dequant()) / d
    lo = GRID[np.clip(np.searchsorted(GRID, mag, side="right") - 1, 0, 7)]
    hi = GRID[np.clip(np.searchsorted(GRID, mag, side="right"), 0, 7)]
    close = lambda a, b: np.abs(a - b) <= 1e-6 * np.maximum(1.0, b)
    assert np.all(close(q, lo) | close(q, hi))
    # signs follow y (zeros keep the sign bit)
    codes = _unpack(v.codes)
    assert np.all((codes >= 8) == np.signbit(y.astype(np.float32)))


def test_unbiased_over_2048_seeds():
    """The binary32 SR quantizer is unbiased up to binary32 rounding of d, 1/d and |y|*r (relative
    2^-23, far below what 2048 seeds resolve): the strict per-coordinate bar on 2048
    coordinates, one of them an outlier."""
    x, xd = _bias_inputs()
    z, rel_bias, rel_noise = _mean_stats(lambda s: O.unrotate(O.sr(x, s, 7, "row").dequant(), s), xd, 2048)
    strict_unbiased(z, "SR baseline (binary32)")


def test_agrees_with_fp64_baseline():
    rng = np.random.default_rng(4)
    x = _bf16(rng.standard_normal((16, 1024)))
    for seed in (1, 2):
        a = O.sr(x, seed, 7, "row").dequant()
        b = O.sr_dequant(x, seed, 7, "row")
        differ = ~np.isclose(a, b, rtol=1e-6, atol=0.0)
        assert np.mean(differ) < 1e-3, np.mean(differ)


def test_mse_ratio_to_msedEN():
    rng = np.random.default_rng(8)
    x = _bf16(rng.standard_normal((64, 1024)))
    mse_e = mse_s = 0.0
    for seed in range(4):
        y = _rotated(x, seed).astype(np.float64)
        mse_e += np.mean((O.msedEN(x, seed, 1, "row").dequant() - y) ** 2)
        mse_s += np.mean((O.sr(x, seed, 7, "row").dequant() - y) ** 2)
    assert mse_s / mse_e >= 1.8, mse_s / mse_e


def test_zero_and_tiny():
    z = O.sr(_bf16(np.zeros((4, 128))), 0, 7, "row")
    assert z.g == 1.0 and np.all(z.scales == 0) and np.all((z.codes & 0x77) == 0)
    xf = np.full((4, 128), 1.0, np.float32)
    xf[1] = 1e-33
    t = O.sr(_bf16(xf), 0, 7, "row")
    assert np.all(t.scales[1] == 0) and np.all(t.scales[0] > 0)
    assert np.all((t.codes[1] & 0x77) == 0)


def test_col_view_is_row_view_of_transpose():
    rng = np.random.default_rng(6)
    x = _bf16(rng.standard_normal((256, 384)))
    a = O.sr(x, 3, 9, "col")
    b = O.sr(_bf16(x.float().numpy().T.copy()), 3, 9, "row")
    assert np.array_equal(a.codes, b.codes) and np.array_equal(a.scales, b.scales) and a.g == b.g
