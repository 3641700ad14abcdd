"""Pins of the oracle's forward quantizer: RTN onto E2M1 in 1x16 groups with the 4/6 grid
choice (CPU only).

Independent checks: a brute-force fp64 re-derivation of both candidates whose roundings come
from library casts (torch float8_e4m3fn, ml_dtypes float4_e2m1fn); the invariant that the
pick never raises the group error; exact round trips on representable inputs.
"""
import ml_dtypes
import numpy as np
import torch

import oracle as O


def _bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16)


def _groups(seed=0, n=512):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((n, 16)).astype(np.float32)
    x[::7] *= 1e-3
    x[::11, 3] *= 40.0              # a group outlier
    x[5] = 0.0                      # an all-zero group
    x[6, :8] = -0.0
    x[13] = rng.integers(-4, 5, 16)  # small integers (exact candidates)
    return _bf16(x.reshape(-1, 64))  # rows of 4 groups


def _library_candidate(xg: np.ndarray, g: np.float32, k: float):
    """Candidate k of one group in fp64 with library roundings: scale via torch's E4M3 cast,
    elements via ml_dtypes' E2M1 cast of x * (1/d) evaluated in fp32."""
    a = np.float32(np.max(np.abs(xg)))
    t = np.float32(a / np.float32(g * np.float32(k)))
    s = torch.tensor([float(t)]).to(torch.float8_e4m3fn)
    sval = np.float32(s.float().item())
    d = np.float32(sval * g)
    if d == 0:
        codes = np.where(np.signbit(xg), 8, 0).astype(np.uint8)
        deq = np.zeros(16)
    else:
        r = np.float32(np.float32(1.0) / d)
        q = (xg * r).astype(np.float32)
        codes = q.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
        deq = q.astype(ml_dtypes.float4_e2m1fn).astype(np.float64) * float(d)
    sse = float(np.sum((xg.astype(np.float64) - deq) ** 2))
    return codes, int(s.view(torch.uint8).item()), sse


def _unpack(codes_row: np.ndarray) -> np.ndarray:
    out = np.empty(codes_row.size * 2, np.uint8)
    out[0::2] = codes_row & 15
    out[1::2] = codes_row >> 4
    return out


def test_pick_never_raises_group_error():
    x = _groups()
    v = O.fwd46(x)
    e6, e4 = v.err6, v.err4
    chosen = np.where(v.choice == 4, e4, e6)
    assert np.array_equal(chosen, np.minimum(e4, e6))
    assert np.all(chosen <= e6)
    ties = e4 == e6
    assert np.all(v.choice[ties] == 6)
    assert (v.choice == 4).any() and (v.choice == 6).any()


def test_candidates_match_library_rederivation():
    x = _groups(1)
    xf = x.float().numpy()
    v = O.fwd46(x)
    g = np.float32(np.max(np.abs(xf)) / np.float32(1792.0))
    assert v.g == g
    R, C = xf.shape
    codes = np.stack([_unpack(r) for r in v.codes])
    agree = 0
    for r in range(R):
        for q in range(C // 16):
            xg = xf[r, 16 * q:16 * q + 16]
            c6, s6, sse6 = _library_candidate(xg, g, 6.0)
            c4, s4, sse4 = _library_candidate(xg, g, 4.0)
            got_c, got_s = codes[r, 16 * q:16 * q + 16], v.scales[r, q]
            if v.choice[r, q] == 6:
                assert np.array_equal(got_c, c6) and got_s == s6
                ok = sse6 <= sse4 * (1 + 1e-5) + 1e-30
            else:
                assert np.array_equal(got_c, c4) and got_s == s4
                ok = sse4 <= sse6 * (1 + 1e-5) + 1e-30
            assert ok, (r, q, sse6, sse4)
            # the oracle's fp32 tree errors agree with the fp64 SSEs
            assert abs(float(v.err6[r, q]) - sse6) <= 1e-5 * sse6 + 1e-38
            assert abs(float(v.err4[r, q]) - sse4) <= 1e-5 * sse4 + 1e-38
            agree += 1
    assert agree == R * C // 16


def test_zero_and_signed_zero_groups():
    x = np.zeros((2, 32), np.float32)
    x[0, 16:] = np.linspace(-1, 1, 16)
    x[1, :16] = -0.0
    v = O.fwd46(_bf16(x))
    assert v.scales[1, 0] == 0 and v.scales[0, 0] == 0
    assert np.all(_unpack(v.codes[1])[:16] == 8)   # -0 keeps its sign
    assert np.all(_unpack(v.codes[0])[:16] == 0)
    vz = O.fwd46(_bf16(np.zeros((1, 32), np.float32)))
    assert vz.g == 1.0 and np.all(vz.scales == 0) and np.all(vz.codes == 0)


def test_representable_inputs_round_trip_exactly():
    """With tensor max A = 1792 * 2^-12 the tensor scale is g = 2^-12 exactly, and a group
    whose max is A has the 4-grid scale t = A/(4g) = 448, an E4M3 value; a group made of
    4-grid values times A/4 is then quantized with zero error, so the 4/6 check must pick the
    4-grid and the dequantized tensor equals the input exactly."""
    rng = np.random.default_rng(4)
    mags4 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0])
    R, C = 8, 64
    vals = mags4[rng.integers(0, 7, (R, C))] * rng.choice([-1, 1], (R, C))
    vals[:, ::16] = 4.0   # every group reaches the top of the 4-grid
    A = 1792.0 * 2.0 ** -12
    x = _bf16(vals * (A / 4))
    v = O.fwd46(x)
    assert v.g == np.float32(2.0 ** -12)
    assert np.all(v.choice == 4) and np.all(v.err4 == 0)
    deq = v.dequant()
    assert np.array_equal(deq, x.float().numpy().astype(np.float64))


def test_dequant_error_is_small_on_gaussian():
    rng = np.random.default_rng(5)
    x = _bf16(rng.standard_normal((64, 256)))
    v = O.fwd46(x)
    xf = x.float().numpy().astype(np.float64)
    rel = np.linalg.norm(v.dequant() - xf) / np.linalg.norm(xf)
    assert 0.03 < rel < 0.12          # 4-bit RTN with 1x16 FP8 scales: ~8-9% relative error
