"""Pins of the oracle's 128-point randomized Hadamard rotation (CPU only)."""
import numpy as np

import oracle as O


def test_dense_hadamard_is_orthogonal():
    H = O.hadamard128()
    assert np.array_equal(np.abs(H), np.ones((128, 128)))
    assert np.array_equal(H @ H.T, 128.0 * np.eye(128))
    assert np.array_equal(H, H.T)
    # Sylvester recursion H_2n = [[H, H], [H, -H]]
    h64 = H[:64, :64]
    assert np.array_equal(H[:64, 64:], h64) and np.array_equal(H[64:, :64], h64) and np.array_equal(H[64:, 64:], -h64)


def test_fwht_of_unit_vectors_are_hadamard_columns():
    H = O.hadamard128()
    for i in range(128):
        e = np.zeros(128, np.float32)
        e[i] = 1.0
        assert np.array_equal(O.fwht128(e).astype(np.float64), H[:, i])


def test_fwht_matches_dense_fp64_within_rounding():
    H = O.hadamard128()
    rng = np.random.default_rng(0)
    for trial in range(200):
        scale = 10.0 ** rng.uniform(-6, 3)
        x = (rng.standard_normal(128) * scale).astype(np.float32)
        if trial % 3 == 0:
            x[rng.integers(0, 128, 3)] *= 50
        y = O.fwht128(x).astype(np.float64)
        ref = H @ x.astype(np.float64)
        # each of the 7 butterfly stages rounds once: |err| <= 7 * 2^-24 * sum|x| (generous)
        bound = 7 * 2.0 ** -24 * np.abs(x.astype(np.float64)).sum() * 1.01
        assert np.max(np.abs(y - ref)) <= bound
        # Parseval for the unnormalised transform: ||Hx||^2 = 128 ||x||^2
        assert abs((y ** 2).sum() - 128 * (x.astype(np.float64) ** 2).sum()) <= 1e-5 * 128 * (x.astype(np.float64) ** 2).sum()


def test_fwht_is_exact_on_small_integers():
    H = O.hadamard128()
    rng = np.random.default_rng(1)
    x = rng.integers(-1000, 1000, 128).astype(np.float32)
    assert np.array_equal(O.fwht128(x).astype(np.float64), H @ x.astype(np.float64))


def test_rotation_cancels_in_products():
    """The shared rotation cancels in an inner product up to the factor 128:
    <H D a, H D b> = 128 <a, b> (why the GEMM of two rotated operands uses alpha = 2^-7)."""
    H = O.hadamard128()
    D = np.diag(O.rht_signs(7).astype(np.float64))
    rng = np.random.default_rng(2)
    a, b = rng.standard_normal(128), rng.standard_normal(128)
    assert abs((H @ D @ a) @ (H @ D @ b) * 2.0 ** -7 - a @ b) < 1e-10
