"""Pins for the calibration oracle (CPU only).

Smoothing factors and the activation scale against their closed forms; the
randomized rank-r factorization against exact properties: an exactly rank-r
matrix is reproduced, the approximation error reaches the Eckart-Young
optimum of the exact SVD (a library routine used only as the check) when the
spectrum has a gap, the factors carry the sign convention, and the result
does not depend on the test matrix beyond rounding.
"""
import numpy as np

from oracle import calibrate as OC


def test_smoothing_closed_form_and_zero_columns():
    x = np.array([[1.0, -4.0, 0.0, 2.0], [-3.0, 1.0, 0.0, 0.5]], np.float32)
    W = np.array([[0.25, 1.0, 2.0, 0.0], [-0.5, -0.25, 1.0, 0.0]], np.float32)
    lam = OC.smoothing_factors(x, W)
    assert lam.dtype == np.float32
    assert lam[0] == np.float32(np.sqrt(np.float32(3.0 / 0.5)))
    assert lam[1] == np.float32(2.0)              # sqrt(4 / 1)
    assert lam[2] == 1.0 and lam[3] == 1.0       # an all-zero column in x or in W
    s_a = OC.act_scale(x, lam)
    want = np.float32(np.max(np.abs(x * (np.float32(1) / lam)[None, :])) / np.float32(2688))
    assert s_a == want
    assert OC.act_scale(np.zeros((2, 4), np.float32), lam) == 1.0


def _spectrum_matrix(rng, K, N, svals):
    U, _ = np.linalg.qr(rng.standard_normal((K, len(svals))))
    V, _ = np.linalg.qr(rng.standard_normal((N, len(svals))))
    return (U * np.asarray(svals)[None, :]) @ V.T


def test_exact_rank_r_matrix_is_reproduced():
    rng = np.random.default_rng(41)
    K, N, r = 96, 160, 8
    A = _spectrum_matrix(rng, K, N, np.linspace(10, 1, r))
    L1, L2 = OC.lowrank_factors(A, r, rng.standard_normal((N, r + 8)), power_iters=2)
    assert np.allclose(L1 @ L2, A, atol=1e-10 * np.abs(A).max())


def test_reaches_the_eckart_young_optimum_with_a_gap():
    rng = np.random.default_rng(42)
    K, N, r = 120, 200, 10
    svals = np.concatenate([np.linspace(50, 20, r), np.linspace(1.0, 0.1, 60)])
    A = _spectrum_matrix(rng, K, N, svals)
    L1, L2 = OC.lowrank_factors(A, r, rng.standard_normal((N, r + 8)), power_iters=4)
    best = np.sqrt(np.sum(np.linalg.svd(A, compute_uv=False)[r:] ** 2))
    assert np.linalg.norm(A - L1 @ L2) <= best * (1 + 1e-9)


def test_sign_convention_and_independence_of_the_test_matrix():
    rng = np.random.default_rng(43)
    K, N, r = 80, 120, 6
    svals = np.concatenate([np.linspace(40, 15, r), np.linspace(1.0, 0.1, 30)])
    A = _spectrum_matrix(rng, K, N, svals)
    L1a, L2a = OC.lowrank_factors(A, r, rng.standard_normal((N, r + 8)), power_iters=6)
    L1b, L2b = OC.lowrank_factors(A, r, rng.standard_normal((N, r + 8)), power_iters=6)
    for t in range(r):
        col = L1a[:, t]
        assert col[np.argmax(np.abs(col))] > 0
    assert np.allclose(L1a, L1b, atol=1e-8 * np.abs(L1a).max())
    assert np.allclose(L2a, L2b, atol=1e-8)
    # L2's rows are orthonormal; L1's columns carry the singular values in descending order
    assert np.allclose(L2a @ L2a.T, np.eye(r), atol=1e-12)
    norms = np.linalg.norm(L1a, axis=0)
    assert np.all(np.diff(norms) < 0) and np.allclose(norms, svals[:r], rtol=1e-9)
