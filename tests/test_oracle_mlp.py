"""Pins for the GELU-MLP oracle (CPU only).

GELU against standard normal table values and two identities of v * Phi(v);
the fused re-quantization against closed-form compositions (zero 4-bit
weights make the up layer's output its bias exactly; dyadic smoothing makes
the down layer's scaling exact); the whole MLP against a brute-force loop on
a tiny shape using Python's own math.erf.
"""
import math
import os

import numpy as np
from scipy.optimize import brentq
from scipy.stats import norm

import workloads as wl
from oracle.calibrate import smoothing_factors
from oracle import formats as F
from oracle import mlp as OM
from oracle import svdq as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "normal_cdf_points.txt")


def _cdf_points():
    v, p = np.loadtxt(GOLDEN, comments="#", unpack=True)
    return np.concatenate([v, -v[1:]]), np.concatenate([p, 1.0 - p[1:]])


def test_gelu_is_v_times_table_phi():
    v, phi = _cdf_points()
    assert np.allclose(OM.gelu(v), v * phi, rtol=0, atol=2e-16)


def test_gelu_odd_part_is_identity():
    """GELU(v) - GELU(-v) = v, since erf is odd: catches a sign or a
    missing 1/2 anywhere in the formula."""
    v = np.linspace(-9, 9, 1001)
    assert np.allclose(OM.gelu(v) - OM.gelu(-v), v, rtol=0, atol=1e-14)
    assert OM.gelu(0.0) == 0.0
    big = np.array([12.0, 30.0])
    assert np.array_equal(OM.gelu(big), big) and np.all(OM.gelu(-big) == 0)


def test_gelu_minimum_location():
    """d/dv [v Phi(v)] = Phi(v) + v phi(v) vanishes at the minimum (about
    v = -0.7518, GELU = -0.17); located with the library's normal pdf/cdf."""
    vstar = brentq(lambda v: norm.cdf(v) + v * norm.pdf(v), -1.5, -0.3, xtol=1e-14)
    g = OM.gelu(np.array([vstar - 1e-4, vstar, vstar + 1e-4]))
    assert g[1] < g[0] and g[1] < g[2]
    assert abs(vstar + 0.7518) < 1e-4 and abs(g[1] + 0.16997) < 1e-5


def _zero_up_layer(K, N, bias, r=32):
    """An up layer with W = 0 and L1 = L2 = 0: its output is the bias exactly."""
    W = np.zeros((N, K), np.float32)
    lam = np.ones(K, np.float32)
    L1 = np.zeros((K, r), np.float32)
    L2 = np.zeros((r, N), np.float32)
    pw = O.pack_weights("nvfp4", W, lam, L1, L2)
    return pw, L1, L2


def test_requantize_of_bias_only_up_layer():
    """v = b exactly, so h = b Phi(b) from the table; h_hat = h * 2^k exactly
    (dyadic inverse smoothing on the down layer's input channels)."""
    rng = np.random.default_rng(21)
    M, K, N = 4, 64, 64
    v_tab, phi_tab = _cdf_points()
    idx = rng.integers(0, len(v_tab), N)
    b = v_tab[idx].astype(np.float32)
    pw, L1, L2 = _zero_up_layer(K, N, b)
    _, x = wl.to_bf16(rng.standard_normal((M, K)).astype(np.float32))
    act = O.quantize_activations("nvfp4", x, pw["inv_lam"], np.float32(0.01))
    v = OM.up_output_f64(act, pw, L1, L2, b)
    assert np.array_equal(v, np.broadcast_to(b.astype(np.float64), (M, N)))
    inv_lam_d = (2.0 ** rng.integers(-3, 4, N)).astype(np.float32)
    s_d = np.float32(2.0 ** -9)
    got = OM.gelu_requantize(v, inv_lam_d, s_d)
    want_h_hat = (b.astype(np.float64) * phi_tab[idx]) * inv_lam_d.astype(np.float64)
    assert np.allclose(got["x_hat"], np.broadcast_to(want_h_hat, (M, N)), rtol=0, atol=1e-15)
    codes, scales = O.nvfp4_quantize(np.broadcast_to(want_h_hat.astype(np.float32), (M, N)), s_d)
    assert np.array_equal(got["codes"], codes) and np.array_equal(got["scales"], scales)
    # the low-rank slot of the down layer: dyadic L1 makes u exact
    r = 32
    L1_d = rng.integers(-2, 3, (N, r)).astype(np.float32) * np.float32(2 ** -4)
    s_w = np.float32(2.0 ** -7)
    la = OM.lora_act(got["x_hat"], L1_d, s_d, s_w)
    u = np.array([[sum(float(got["x_hat"][m, n]) * float(L1_d[n, t]) for n in range(N)) for t in range(r)]
                  for m in range(M)])
    assert np.allclose(la, u / (float(s_d) * float(s_w)), rtol=1e-13, atol=0)


def test_gelu_applies_before_smoothing_and_after_bias():
    """Exchanging any two of (bias, GELU, smoothing) changes the result on
    this input: the order is bias -> GELU -> times inv_lambda."""
    v = np.tile(np.array([[-1.0, 0.5, 2.0, -2.5]]), (1, 4))
    inv = np.tile(np.array([4.0, 0.25, 2.0, 0.5], np.float32), 4)
    got = OM.gelu_requantize(v, inv, np.float32(1e-3))["x_hat"]
    assert np.allclose(got, OM.gelu(v) * inv, rtol=0, atol=0)
    assert not np.allclose(got, OM.gelu(v * inv))


def test_mlp_matches_brute_force_loops():
    """A tiny MLP: every step written out as Python loops with math.erf."""
    rng = np.random.default_rng(22)
    M, K, N, Nd, r = 2, 64, 32, 16, 4
    _, x = wl.to_bf16(rng.standard_normal((M, K)).astype(np.float32))
    _, Wu = wl.to_bf16(rng.standard_normal((N, K)).astype(np.float32) * 0.1)
    _, L1u = wl.to_bf16(rng.standard_normal((K, r)).astype(np.float32) * 0.1)
    _, L2u = wl.to_bf16(rng.standard_normal((r, N)).astype(np.float32) * 0.1)
    bu = wl.to_bf16(rng.standard_normal(N).astype(np.float32) * 0.3)[1]
    lam_u = smoothing_factors(x, Wu)
    _, Wd = wl.to_bf16(rng.standard_normal((Nd, N)).astype(np.float32) * 0.1)
    _, L1d = wl.to_bf16(rng.standard_normal((N, r)).astype(np.float32) * 0.1)
    _, L2d = wl.to_bf16(rng.standard_normal((r, Nd)).astype(np.float32) * 0.1)
    bd = wl.to_bf16(rng.standard_normal(Nd).astype(np.float32) * 0.3)[1]
    lam_d = np.exp(rng.uniform(-1, 1, N)).astype(np.float32)
    pw_u = O.pack_weights("nvfp4", Wu, lam_u, L1u, L2u)
    pw_d = O.pack_weights("nvfp4", Wd, lam_d, L1d, L2d)
    act_u = O.quantize_activations("nvfp4", x, pw_u["inv_lam"], np.float32(0.002))
    s_d = np.float32(0.001)
    y, act_d, v = OM.mlp_f64(act_u, pw_u, L1u, L2u, bu, pw_d, L1d, L2d, bd, s_d)

    def deq(codes, scales, s, row, k):
        return F.E2M1_VALUE[codes[row, k]] * F.E4M3_VALUE[scales[row, k // 16]] * float(s)

    h_hat = np.zeros((M, N))
    for m in range(M):
        for n in range(N):
            acc = sum(deq(act_u["codes"], act_u["scales"], act_u["s_a"], m, k) *
                      deq(pw_u["codes"], pw_u["scales"], pw_u["s_w"], n, k) for k in range(K))
            for t in range(r):
                acc += sum(float(act_u["x_hat"][m, k]) * float(L1u[k, t]) for k in range(K)) * float(L2u[t, n])
            acc += float(bu[n])
            assert abs(acc - v[m, n]) <= 1e-12 * (1 + abs(acc))
            h = 0.5 * acc * (1.0 + math.erf(acc / math.sqrt(2.0)))
            h_hat[m, n] = h * float(pw_d["inv_lam"][n])
    assert np.allclose(act_d["x_hat"], h_hat, rtol=1e-12, atol=1e-15)
    for m in range(M):
        for j in range(Nd):
            acc = sum(deq(act_d["codes"], act_d["scales"], s_d, m, n) *
                      deq(pw_d["codes"], pw_d["scales"], pw_d["s_w"], j, n) for n in range(N))
            for t in range(r):
                acc += sum(h_hat[m, n] * float(L1d[n, t]) for n in range(N)) * float(L2d[t, j])
            acc += float(bd[j])
            assert abs(acc - y[m, j]) <= 1e-10 * (1 + abs(acc)), (m, j, acc, y[m, j])
