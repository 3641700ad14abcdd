"""Pins of the oracle's GEMM by dequantization and of the composed linear layer (CPU only).

Independent checks: closed-form products; an exactly representable forward case equal to
the unquantized product; the synthetic Fig. 9 experiment -- the relative squared error of the
mean of B quantized backward products against the unquantized product falls like 1/B for
MS-EDEN (unbiased) and plateaus for a biased scheme.
"""
import numpy as np
import torch

import oracle as O


def _bf16(a) -> torch.Tensor:
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16)


def test_gemm_closed_forms():
    rng = np.random.default_rng(0)
    A = rng.standard_normal((5, 7))
    # identity operand: C = alpha * A I^T = alpha A
    assert np.array_equal(O.gemm(A, np.eye(7), 2.0), 2.0 * A)
    # integer matrices: exact in fp64, checked against an explicit double loop here
    Ai = rng.integers(-9, 10, (6, 8)).astype(np.float64)
    Bi = rng.integers(-9, 10, (3, 8)).astype(np.float64)
    C = O.gemm(Ai, Bi)
    for i in range(6):
        for j in range(3):
            assert C[i, j] == sum(Ai[i, k] * Bi[j, k] for k in range(8))


def test_forward_exact_case_equals_unquantized_product():
    """Inputs on the 4-grid times A/4 with A = 1792*2^-12 quantize exactly (see the forward
    quantizer pins), so the forward GEMM equals X W^T."""
    rng = np.random.default_rng(1)
    mags4 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0])

    def exact(R, C):
        v = mags4[rng.integers(0, 7, (R, C))] * rng.choice([-1, 1], (R, C))
        v[:, ::16] = 4.0
        return _bf16(v * (1792.0 * 2.0 ** -12 / 4))

    x, w = exact(32, 128), exact(48, 128)
    y, vx, vw = O.linear_fwd(x, w)
    ref = x.float().numpy().astype(np.float64) @ w.float().numpy().astype(np.float64).T
    assert np.array_equal(y, ref)


def test_forward_error_is_small():
    rng = np.random.default_rng(2)
    x = _bf16(rng.standard_normal((64, 256)))
    w = _bf16(rng.standard_normal((96, 256)) * 0.02)
    y, _, _ = O.linear_fwd(x, w)
    ref = x.float().numpy().astype(np.float64) @ w.float().numpy().astype(np.float64).T
    rel = np.linalg.norm(y - ref) / np.linalg.norm(ref)
    assert rel < 0.15


def _fig9_curve(make_dx, ref, Bs):
    acc = np.zeros_like(ref)
    out = {}
    n = 0
    for B in Bs:
        while n < B:
            acc += make_dx(n)
            n += 1
        out[B] = np.linalg.norm(acc / n - ref) ** 2 / np.linalg.norm(ref) ** 2
    return out


def test_synthetic_fig9_dgrad_unbiased():
    """Relative squared error of the mean of B MS-EDEN dgrad products vs B: slope ~ -1 in log-log
    (unbiased); a biased backward (the forward RTN + 4/6 quantizer, deterministic) plateaus."""
    rng = np.random.default_rng(3)
    M, N, K = 64, 256, 128
    dy = _bf16(rng.standard_normal((M, N)))
    w = _bf16(rng.standard_normal((N, K)) * 0.02)
    ref = dy.float().numpy().astype(np.float64) @ w.float().numpy().astype(np.float64)

    def eden_dx(i):
        seed = 100 + i
        a = O.msedEN(dy, seed, O.TID_DY_ROW, "row")
        b = O.msedEN(w, seed, O.TID_W_COL, "col")
        return O.gemm_views(a, b, 2.0 ** -7)

    Bs = [1, 4, 16, 64, 256, 1024]
    curve = _fig9_curve(eden_dx, ref, Bs)
    slope = np.polyfit(np.log(Bs), np.log([curve[B] for B in Bs]), 1)[0]
    assert -1.2 < slope < -0.8, (slope, curve)

    # biased control: forward quantizer on dY (rows) and W^T (rows) -- no randomness at all
    a46 = O.fwd46(dy)
    b46 = O.fwd46(torch.from_numpy(np.ascontiguousarray(w.float().numpy().T)).to(torch.bfloat16))
    biased = O.gemm_views(a46, b46, 1.0)
    err_biased = np.linalg.norm(biased - ref) ** 2 / np.linalg.norm(ref) ** 2
    assert curve[1024] < err_biased / 50


def test_linear_bwd_views_and_alpha():
    """The composed backward: dX and dW agree with the unquantized products within the
    single-sample error, and dW uses the column views of dY and X."""
    rng = np.random.default_rng(4)
    M, K, N = 128, 128, 256
    x = _bf16(rng.standard_normal((M, K)))
    w = _bf16(rng.standard_normal((N, K)) * 0.02)
    dy = _bf16(rng.standard_normal((M, N)))
    dx, dw, views = O.linear_bwd(dy, x, w, seed=5)
    X, W, DY = (t.float().numpy().astype(np.float64) for t in (x, w, dy))
    for got, ref in ((dx, DY @ W), (dw, DY.T @ X)):
        rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
        assert rel < 0.2, rel
    assert views["dy_col"].shape == (N, M) and views["x_col"].shape == (K, M)
    assert views["dy_row"].shape == (M, N) and views["w_col"].shape == (K, N)
