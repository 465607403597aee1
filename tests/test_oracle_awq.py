"""Pins for the AWQ W4A16 oracle (CPU only)."""
import numpy as np

import workloads as wl
from oracle import awq as A
from oracle import formats as F


def test_awq_codes_range_and_error_bound():
    rng = np.random.default_rng(21)
    _, W = wl.to_bf16(rng.standard_normal((32, 256)).astype(np.float32) * 0.02)
    q, sc, z = A.awq_quantize(W)
    assert q.min() >= 0 and q.max() <= 15 and z.min() >= 0 and z.max() <= 15
    err = np.abs(W.astype(np.float64) - A.awq_dequantize(q, sc, z))
    # inside [mn, mx] the grid step is sc; bf16 rounding of sc shifts the
    # top of the grid by at most 15 * sc * 2^-8
    bound = np.repeat(sc.astype(np.float64), 64, axis=1) * (0.5 + 15 * 2 ** -8) + 1e-12
    assert np.all(err <= bound)


def test_awq_on_grid_round_trip():
    rng = np.random.default_rng(22)
    N, K = 8, 128
    q = rng.integers(0, 16, (N, K)).astype(np.uint8)
    qg = q.reshape(N, K // 64, 64)
    qg[:, :, 0] = 0
    qg[:, :, 1] = 15
    z = rng.integers(1, 15, (N, K // 64)).astype(np.uint8)
    sc = F.bf16_round((2.0 ** rng.integers(-9, -3, (N, K // 64))).astype(np.float32))
    W = ((qg.astype(np.float32) - z[:, :, None]) * sc[:, :, None]).reshape(N, K).astype(np.float32)
    q2, sc2, z2 = A.awq_quantize(W)
    assert np.array_equal(sc2, sc) and np.array_equal(z2, z) and np.array_equal(q2, q)


def test_awq_constant_and_zero_groups():
    W = np.zeros((3, 64), np.float32)
    W[1] = 0.5
    W[2] = -0.25
    q, sc, z = A.awq_quantize(W)
    deq = A.awq_dequantize(q, sc, z)
    assert np.all(deq[0] == 0)
    assert np.allclose(deq[1], 0.5, rtol=2 ** -7)
    assert np.allclose(deq[2], -0.25, rtol=2 ** -7)


def test_awq_linear_matches_brute_force_gemv():
    rng = np.random.default_rng(23)
    M, N, K = 2, 6, 128
    _, x = wl.to_bf16(rng.standard_normal((M, K)).astype(np.float32))
    _, W = wl.to_bf16(rng.standard_normal((N, K)).astype(np.float32) * 0.02)
    _, b = wl.to_bf16(rng.standard_normal(N).astype(np.float32) * 0.01)
    q, sc, z = A.awq_quantize(W)
    y, y64 = A.awq_linear(x, q, sc, z, b)
    for m in range(M):
        for n in range(N):
            acc = float(b[n])
            for k in range(K):
                acc += float(x[m, k]) * (int(q[n, k]) - int(z[n, k // 64])) * float(sc[n, k // 64])
            assert abs(acc - y64[m, n]) <= 1e-12 * (1 + abs(acc))
    assert np.array_equal(y, F.bf16_round(y64.astype(np.float32)))
