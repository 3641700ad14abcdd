"""Pins of the oracle's square-block forward quantizer (one E4M3 scale per 16x16 block, RTN with
the 4/6 choice per block) and of its column view (CPU only).

Independent checks: blocks made of one repeated row reduce to the pinned 1x16 quantizer (their
block max is the row max and the block error is exactly 16 times the row error); a brute-force
fp64 re-derivation of both candidates of every block with library roundings (torch's E4M3 cast,
ml_dtypes' E2M1 cast); the column view dequantizes to the exact transpose; a block's result
depends on its own elements and the tensor scale only.
"""
import ml_dtypes
import numpy as np
import torch

import oracle as O


def _bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16)


def _matrix(seed, R=64, C=96):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((R, C)).astype(np.float32)
    x[:16, :16] *= 1e-3                 # a quiet block
    x[16:32, 32:48] *= 30.0             # a loud block
    x[R - 24, C - 26] = 250.0           # a single outlier in its block
    x[R - 16:, C - 16:] = 0.0           # an all-zero block
    return x


def _unpack(codes: np.ndarray) -> np.ndarray:
    out = np.empty((codes.shape[0], codes.shape[1] * 2), np.uint8)
    out[:, 0::2] = codes & 15
    out[:, 1::2] = codes >> 4
    return out


def test_repeated_rows_reduce_to_group_quantizer():
    rng = np.random.default_rng(3)
    base = rng.standard_normal((4, 128)).astype(np.float32)
    base[1] *= 1e-2
    base[2, ::5] *= 20.0
    x = _bf16(np.repeat(base, 16, axis=0))          # block rows of 16 identical rows
    row, _ = O.fwd46_sq(x)
    ref = O.fwd46(x)
    assert row.g == ref.g
    assert np.array_equal(row.codes, ref.codes)
    assert np.array_equal(row.scales, ref.scales)
    assert np.array_equal(row.choice, ref.choice[0::16])
    assert np.array_equal(row.err6, ref.err6[0::16] * np.float32(16))


def _library_block(xb: np.ndarray, g: np.float32, k: float):
    a = np.float32(np.max(np.abs(xb)))
    t = np.float32(a / np.float32(g * np.float32(k)))
    s = torch.tensor([float(t)]).to(torch.float8_e4m3fn)
    d = np.float32(np.float32(s.float().item()) * g)
    if d == 0:
        codes = np.where(np.signbit(xb), 8, 0).astype(np.uint8)
        deq = np.zeros_like(xb, dtype=np.float64)
    else:
        r = np.float32(np.float32(1.0) / d)
        q = (xb * r).astype(np.float32)
        codes = q.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
        deq = q.astype(ml_dtypes.float4_e2m1fn).astype(np.float64) * float(d)
    return codes, int(s.view(torch.uint8).item()), float(np.sum((xb.astype(np.float64) - deq) ** 2))


def test_blocks_match_library_rederivation():
    x = _bf16(_matrix(1))
    xf = x.float().numpy()
    row, col = O.fwd46_sq(x)
    g = np.float32(np.max(np.abs(xf)) / np.float32(1792.0))
    assert row.g == g and col.g == g
    codes = _unpack(row.codes)
    R, C = xf.shape
    for rb in range(R // 16):
        for q in range(C // 16):
            xb = xf[16 * rb:16 * rb + 16, 16 * q:16 * q + 16]
            c6, s6, e6 = _library_block(xb, g, 6.0)
            c4, s4, e4 = _library_block(xb, g, 4.0)
            pick = row.choice[rb, q]
            c, s = (c6, s6) if pick == 6 else (c4, s4)
            assert np.array_equal(codes[16 * rb:16 * rb + 16, 16 * q:16 * q + 16], c), (rb, q)
            assert np.all(row.scales[16 * rb:16 * rb + 16, q] == s), (rb, q)
            mine, other = (e6, e4) if pick == 6 else (e4, e6)
            assert mine <= other * (1 + 1e-5) + 1e-30, (rb, q, e6, e4)
            assert abs(float(row.err6[rb, q]) - e6) <= 1e-5 * e6 + 1e-38
            assert abs(float(row.err4[rb, q]) - e4) <= 1e-5 * e4 + 1e-38
    assert (row.choice == 4).any() and (row.choice == 6).any()


def test_column_view_is_the_transpose():
    x = _bf16(_matrix(2, 48, 64))   # R = 48, C = 64
    row, col = O.fwd46_sq(x)
    assert col.shape == (64, 48)
    assert np.array_equal(col.dequant(), row.dequant().T)
    assert np.array_equal(O.transpose_codes(col.codes), row.codes)


def test_block_depends_on_its_own_elements_only():
    xf = _matrix(5)
    A = float(np.max(np.abs(xf)))
    y = xf.copy()
    y[0, 0] = 0.75 * A                    # change one element of block (0, 0) only
    r1, _ = O.fwd46_sq(_bf16(xf), A=A)
    r2, _ = O.fwd46_sq(_bf16(y), A=A)
    c1, c2 = _unpack(r1.codes), _unpack(r2.codes)
    assert not np.array_equal(r1.scales[:16, 0], r2.scales[:16, 0])
    mask = np.ones(c1.shape, bool)
    mask[:16, :16] = False
    assert np.array_equal(c1[mask], c2[mask])
    assert np.array_equal(r1.scales[:, 1:], r2.scales[:, 1:]) and np.array_equal(r1.scales[16:], r2.scales[16:])


def test_zero_tensor_and_signed_zeros():
    x = np.zeros((16, 32), np.float32)
    x[3, :16] = -0.0
    row, col = O.fwd46_sq(_bf16(x))
    assert row.g == 1.0 and np.all(row.scales == 0) and np.all(col.scales == 0)
    c = _unpack(row.codes)
    assert np.all(c[3, :16] == 8) and np.all(c[:3] == 0)
    assert np.all(row.choice == 6)
