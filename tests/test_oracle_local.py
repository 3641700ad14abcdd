"""Pins of the oracle's CTA-local forward quantizer (one tensor scale per block of 128 rows)
and of its GEMM by dequantization (CPU only).

Independent checks: every row block equals the pinned global quantizer applied to that block
alone (whose tensor max is then the block max); blocks with equal maxima reproduce the global
quantizer; blocks that are power-of-two multiples of one another get identical codes and scales
and exactly scaled tensor scales; a block's result depends on its own rows only.
"""
import numpy as np
import torch

import oracle as O


def _bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16)


def _x(seed, R=512, C=256):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((R, C)).astype(np.float32)
    x[128:256] *= 1e-3           # a quiet block
    if R >= 512:
        x[300, 17] = 400.0        # an outlier in the third block
        x[384:] = 0.0             # an all-zero block
    return _bf16(x)


def test_each_block_is_the_global_quantizer_of_that_block():
    x = _x(0)
    v = O.fwd46_local(x)
    assert v.g.shape == (4,)
    for b in range(4):
        ref = O.fwd46(x[128 * b:128 * b + 128])
        assert v.g[b] == ref.g, b
        assert np.array_equal(v.codes[128 * b:128 * b + 128], ref.codes), b
        assert np.array_equal(v.scales[128 * b:128 * b + 128], ref.scales), b
    assert v.g[3] == 1.0 and np.all(v.scales[384:] == 0)      # the zero block


def test_equal_block_maxima_reproduce_the_global_quantizer():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((256, 128)).astype(np.float32)
    x[0, 0], x[128, 5] = 9.0, -9.0                      # both blocks reach max |x| = 9
    v, ref = O.fwd46_local(_bf16(x)), O.fwd46(_bf16(x))
    assert np.all(v.g == ref.g)
    assert np.array_equal(v.codes, ref.codes) and np.array_equal(v.scales, ref.scales)
    assert np.array_equal(v.dequant(), ref.dequant())


def test_power_of_two_blocks_scale_exactly():
    rng = np.random.default_rng(2)
    base = rng.standard_normal((128, 256)).astype(np.float32)
    x = np.concatenate([base, base * 8.0, base * 0.25])
    v = O.fwd46_local(_bf16(x))
    assert v.g[1] == v.g[0] * 8 and v.g[2] == v.g[0] * 0.25
    for b in (1, 2):
        assert np.array_equal(v.codes[128 * b:128 * b + 128], v.codes[:128])
        assert np.array_equal(v.scales[128 * b:128 * b + 128], v.scales[:128])
    d = v.dequant()
    assert np.array_equal(d[128:256], d[:128] * 8.0) and np.array_equal(d[256:], d[:128] * 0.25)
    rows = np.array([3, 200, 383])
    assert np.array_equal(v.dequant_rows(rows), d[rows])


def test_blocks_are_independent():
    x = _x(3).float().numpy()
    y = x.copy()
    y[130:140] *= 64.0                                  # change the second block only
    a, b = O.fwd46_local(_bf16(x)), O.fwd46_local(_bf16(y))
    keep = np.r_[0:128, 256:512]
    assert np.array_equal(a.codes[keep], b.codes[keep]) and np.array_equal(a.scales[keep], b.scales[keep])
    assert a.g[0] == b.g[0] and a.g[2] == b.g[2] and a.g[1] != b.g[1]


def test_local_gemm_applies_row_and_column_corrections():
    """C = A_hat B_hat^T with each operand's per-block tensor scale as a row (column) factor."""
    va = O.fwd46_local(_x(4, 256, 128))
    vb = O.fwd46_local(_x(5, 384, 128))
    got = O.gemm_views(va, vb)
    A0 = va.dequant() / va.row_g()[:, None]
    B0 = vb.dequant() / vb.row_g()[:, None]
    ref = O.gemm(A0, B0) * np.outer(va.row_g().astype(np.float64), vb.row_g().astype(np.float64))
    bound = O.gemm(np.abs(va.dequant()), np.abs(vb.dequant()))
    assert np.all(np.abs(got - ref) <= 1e-13 * bound)       # fp64 rounding of the two orders only
    # and the factors really differ between blocks (a global g would fail the first check)
    assert len(set(va.g.tolist())) > 1 and len(set(vb.g.tolist())) > 1
