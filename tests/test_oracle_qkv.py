"""Pins for the QKV + RMSNorm + RoPE oracle (CPU only).

RMSNorm against its defining properties (unit mean square with gamma = 1,
invariance to a positive scale of the input, gamma applied per feature);
RoPE against rotation identities (zero angle, a quarter turn, norm
preservation, composition of angles) and Python's complex multiplication;
the composition against a brute-force loop over a tiny layer.
"""
import cmath
import math

import numpy as np

import workloads as wl
from oracle.calibrate import smoothing_factors
from oracle import qkv as OQ
from oracle import svdq as O


def test_rmsnorm_unit_mean_square_and_scale_invariance():
    rng = np.random.default_rng(31)
    u = rng.standard_normal((5, 3, 128)) * 7.0
    n = OQ.rmsnorm(u, np.ones(128), eps=0.0)
    assert np.allclose(np.mean(n * n, axis=-1), 1.0, rtol=1e-14)
    assert np.allclose(OQ.rmsnorm(3.5 * u, np.ones(128), eps=0.0), n, rtol=1e-13)
    g = rng.uniform(0.5, 2.0, 128)
    assert np.allclose(OQ.rmsnorm(u, g, eps=0.0), n * g, rtol=1e-14)


def test_rmsnorm_closed_form_and_eps():
    u = np.zeros(128)
    u[0], u[1] = 3.0, 4.0                 # mean square 25 / 128
    want = u / math.sqrt(25.0 / 128 + 1e-6)
    assert np.allclose(OQ.rmsnorm(u, np.ones(128)), want, rtol=1e-15)
    assert np.all(OQ.rmsnorm(np.zeros(128), np.ones(128)) == 0)   # eps keeps zero finite


def test_rope_rotation_identities():
    rng = np.random.default_rng(32)
    M, d = 4, 128
    u = rng.standard_normal((M, 2, d))
    zero = OQ.rope(u, np.ones((M, d // 2)), np.zeros((M, d // 2)))
    assert np.array_equal(zero, u)
    quarter = OQ.rope(u, np.zeros((M, d // 2)), np.ones((M, d // 2)))
    assert np.array_equal(quarter[..., 0::2], -u[..., 1::2]) and np.array_equal(quarter[..., 1::2], u[..., 0::2])
    phi1, phi2 = rng.uniform(-4, 4, (M, d // 2)), rng.uniform(-4, 4, (M, d // 2))
    r1 = OQ.rope(u, np.cos(phi1), np.sin(phi1))
    pair_norm = lambda x: x[..., 0::2] ** 2 + x[..., 1::2] ** 2
    assert np.allclose(pair_norm(r1), pair_norm(u), rtol=1e-13)
    r12 = OQ.rope(r1, np.cos(phi2), np.sin(phi2))
    assert np.allclose(r12, OQ.rope(u, np.cos(phi1 + phi2), np.sin(phi1 + phi2)), atol=1e-12)


def test_rope_is_complex_multiplication():
    rng = np.random.default_rng(33)
    M, d = 3, 8
    u = rng.standard_normal((M, 1, d))
    phi = rng.uniform(-3, 3, (M, d // 2))
    got = OQ.rope(u, np.cos(phi), np.sin(phi))
    for m in range(M):
        for i in range(d // 2):
            z = complex(u[m, 0, 2 * i], u[m, 0, 2 * i + 1]) * cmath.exp(1j * phi[m, i])
            assert abs(got[m, 0, 2 * i] - z.real) < 1e-14 and abs(got[m, 0, 2 * i + 1] - z.imag) < 1e-14


def test_qkv_layer_matches_brute_force_loops():
    """Two heads of d = 128 (Q | K | V = 768 columns) on 2 tokens."""
    rng = np.random.default_rng(34)
    M, K, H, d, r = 2, 64, 2, 128, 4
    N = 3 * H * d
    _, x = wl.to_bf16(rng.standard_normal((M, K)).astype(np.float32))
    _, W = wl.to_bf16(rng.standard_normal((N, K)).astype(np.float32) * 0.1)
    _, L1 = wl.to_bf16(rng.standard_normal((K, r)).astype(np.float32) * 0.1)
    _, L2 = wl.to_bf16(rng.standard_normal((r, N)).astype(np.float32) * 0.1)
    b = wl.to_bf16(rng.standard_normal(N).astype(np.float32) * 0.1)[1]
    lam = smoothing_factors(x, W)
    gq, gk = rng.uniform(0.5, 1.5, d), rng.uniform(0.5, 1.5, d)
    phi = rng.uniform(-3, 3, (M, d // 2))
    pw = O.pack_weights("nvfp4", W, lam, L1, L2)
    act = O.quantize_activations("nvfp4", x, pw["inv_lam"], np.float32(0.003))
    got = OQ.qkv_layer_f64(act, pw, L1, L2, b, gq, gk, np.cos(phi), np.sin(phi), H)
    v = O.linear_f64("nvfp4", act, pw, L1, L2, b)          # pinned by the layer's own tests
    for m in range(M):
        for part, gamma in ((0, gq), (1, gk), (2, None)):
            for h in range(H):
                c0 = part * H * d + h * d
                u = [float(v[m, c0 + j]) for j in range(d)]
                if gamma is None:
                    want = u
                else:
                    rms = math.sqrt(sum(t * t for t in u) / d + 1e-6)
                    n = [u[j] / rms * float(gamma[j]) for j in range(d)]
                    want = []
                    for i in range(d // 2):
                        z = complex(n[2 * i], n[2 * i + 1]) * cmath.exp(1j * phi[m, i])
                        want += [z.real, z.imag]
                for j in range(d):
                    assert abs(got[m, c0 + j] - want[j]) <= 1e-12 * (1 + abs(want[j])), (m, part, h, j)
