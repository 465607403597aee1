"""Pins for the SVDQuant W4A4 oracle (CPU only).

Every oracle function is tied to something other than itself: closed forms
(an exactly rank-r weight leaves a zero residual; on-grid data is a fixed
point of quantization; on-grid operands make the quantized GEMM exact),
error bounds from the format definitions, and brute-force loops on tiny
shapes.
"""
import numpy as np
import pytest

import workloads as wl
from oracle.calibrate import smoothing_factors
from tests.helpers import svdq_inputs
from oracle import formats as F
from oracle import svdq as O


def _rng(s):
    return np.random.default_rng(s)


# ------------------------------------------------------------ smoothing -----

def test_smoothing_preserves_product_and_scales_columns():
    rng = _rng(1)
    M, K, N = 16, 64, 24
    _, x = wl.to_bf16(rng.standard_normal((M, K)).astype(np.float32) * 3)
    _, W = wl.to_bf16(rng.standard_normal((N, K)).astype(np.float32) * 0.02)
    lam = np.exp(rng.uniform(-2, 2, K)).astype(np.float32)
    inv = O.inverse_smoothing(lam)
    assert np.array_equal(inv, (np.float32(1) / lam).astype(np.float32))
    xh = O.smooth_activations(x, inv)
    Wh = O.smooth_weight(W, lam)
    # input channel j (a column of x and of W) is divided / multiplied by lambda_j
    assert np.allclose(xh[:, 5], x[:, 5] / lam[5], rtol=2 ** -22)
    assert np.allclose(Wh[:, 5], W[:, 5].astype(np.float64) * lam[5], rtol=0)
    ref = x.astype(np.float64) @ W.astype(np.float64).T
    got = xh.astype(np.float64) @ Wh.T
    assert np.max(np.abs(got - ref)) <= 1e-6 * np.max(np.abs(ref))


def test_unit_smoothing_is_identity():
    rng = _rng(2)
    _, x = wl.to_bf16(rng.standard_normal((8, 32)).astype(np.float32))
    xh = O.smooth_activations(x, O.inverse_smoothing(np.ones(32, np.float32)))
    assert np.array_equal(xh, x)


# ------------------------------------------------------------ residual ------

def _dyadic_rank_r(rng, K, N, r):
    """bf16-exact factors whose product is exactly representable in bf16."""
    L1 = rng.integers(-2, 3, (K, r)).astype(np.float32) * np.float32(2 ** -4)
    L2 = rng.integers(-2, 3, (r, N)).astype(np.float32) * np.float32(2 ** -4)
    return L1, L2


def test_exact_rank_r_weight_gives_zero_residual():
    rng = _rng(3)
    K, N, r = 64, 32, 4
    L1, L2 = _dyadic_rank_r(rng, K, N, r)
    lam = (2.0 ** rng.integers(-3, 4, K)).astype(np.float32)     # powers of two keep W exact
    W = ((L1 @ L2).T / lam[None, :]).astype(np.float32)
    assert np.array_equal(F.bf16_round(W), W)
    R = O.residual(W, lam, L1, L2)
    assert np.all(R == 0)
    codes, scales = O.nvfp4_quantize(R, O.nvfp4_tensor_scale(R))
    assert np.all(codes == 0) and np.all(scales == 0)
    q, sc = O.int4_quantize(R)
    assert np.all(q == 0) and np.all(sc == 0)


def test_residual_orientation_and_sign():
    rng = _rng(4)
    K, N, r = 48, 40, 3
    _, W = wl.to_bf16(rng.standard_normal((N, K)).astype(np.float32))
    _, L1 = wl.to_bf16(rng.standard_normal((K, r)).astype(np.float32))
    _, L2 = wl.to_bf16(rng.standard_normal((r, N)).astype(np.float32))
    lam = np.exp(rng.uniform(-1, 1, K)).astype(np.float32)
    R = O.residual(W, lam, L1, L2).astype(np.float64)
    # brute force: R[n,k] = W[n,k]*lam[k] - sum_t L1[k,t] L2[t,n]
    for n, k in [(0, 0), (3, 7), (N - 1, K - 1), (17, 29)]:
        s = sum(float(L1[k, t]) * float(L2[t, n]) for t in range(r))
        want = float(W[n, k]) * float(lam[k]) - s
        assert abs(R[n, k] - want) <= 2 ** -23 * max(abs(want), 1e-30) * 2


# ------------------------------------------------------------ NVFP4 ---------

def _on_grid_nvfp4(rng, rows, K, s):
    """Values that NVFP4 represents exactly with the given power-of-two s,
    each group holding a +-6 so that its scale is recovered exactly."""
    ng = K // 16
    codes = rng.integers(0, 16, (rows, K)).astype(np.uint8)
    pos = rng.integers(0, 16, (rows, ng))
    g = codes.reshape(rows, ng, 16)
    for i in range(rows):
        for j in range(ng):
            g[i, j, pos[i, j]] = 7 | (rng.integers(0, 2) << 3)
    sb = rng.integers(0x10, 0x70, (rows, ng)).astype(np.uint8)     # normal E4M3 scales
    v = F.e2m1_decode(codes).reshape(rows, ng, 16) * F.e4m3_decode(sb)[:, :, None] * s
    return v.reshape(rows, K).astype(np.float32), codes, sb


def test_nvfp4_on_grid_is_fixed_point():
    rng = _rng(5)
    s = np.float32(2.0 ** -9)
    v, codes, sb = _on_grid_nvfp4(rng, 12, 256, s)
    # -0 codes come back as +0 only if the value is +0; on-grid -0 stays -0
    got_codes, got_sb = O.nvfp4_quantize(v, s)
    assert np.array_equal(got_sb, sb)
    assert np.array_equal(got_codes, codes)
    assert np.array_equal(O.nvfp4_dequantize(got_codes, got_sb, s), v.astype(np.float64))


def test_nvfp4_codes_are_nearest_and_bounded():
    rng = _rng(6)
    x = rng.standard_normal((32, 512)).astype(np.float32)
    x[:, rng.choice(512, 5, replace=False)] *= 40
    s = O.nvfp4_tensor_scale(x)
    assert s == np.float32(np.max(np.abs(x)) / np.float32(2688.0))
    codes, sb = O.nvfp4_quantize(x, s)
    d = (F.e4m3_decode(sb).astype(np.float32) * s).astype(np.float32)
    ratio = (x.reshape(32, 32, 16) / d[:, :, None]).astype(np.float64)
    q = F.e2m1_decode(codes).reshape(32, 32, 16)
    grid = np.concatenate([-F.E2M1_MAG[::-1], F.E2M1_MAG])
    # no grid value is strictly closer than the chosen one (|ratio| clipped to 6)
    r = np.clip(ratio, -6, 6)
    best = np.min(np.abs(r[..., None] - grid), axis=-1)
    assert np.all(np.abs(r - q) <= best + 0.0)
    # scale rounding: sb is the nearest E4M3 to a/(6s), so |ratio| <= 6 * t/float(sb) <= 6 (1 + 2^-4)
    assert np.max(np.abs(ratio)) <= 6.0 * (1 + 2 ** -4)
    # the group that holds the tensor max gets the largest scale, 448
    i, j = np.unravel_index(np.argmax(np.abs(x)), x.shape)
    assert sb[i, j // 16] == 0x7E


def test_nvfp4_zero_group_and_signed_zero():
    x = np.zeros((2, 32), dtype=np.float32)
    x[0, 16:] = np.linspace(-1, 1, 16, dtype=np.float32)
    x[0, 16] = -1e-6                                     # rounds to -0 within its group
    s = np.float32(1.0 / 2688.0)
    codes, sb = O.nvfp4_quantize(x, s)
    assert np.all(codes[0, :16] == 0) and sb[0, 0] == 0         # zero group: +0 codes
    assert np.all(codes[1] == 0) and np.all(sb[1] == 0)
    assert (codes[0, 16] >> 3) == 1
    # tiny negative in a group whose scale is set by +-1: -1e-6 / d rounds to -0 -> 0x8
    y = np.array([[1.0] + [-1e-6] * 15], dtype=np.float32)
    c, _ = O.nvfp4_quantize(y, np.float32(1.0 / 2688.0))
    assert np.all(c[0, 1:] == 0x8)


def test_nvfp4_zero_tensor_scale_is_one():
    assert O.nvfp4_tensor_scale(np.zeros((4, 16), np.float32)) == np.float32(1.0)


# ------------------------------------------------------------ INT4 ----------

def test_int4_on_grid_is_fixed_point_and_range():
    rng = _rng(7)
    rows, K = 6, 256
    q = rng.integers(-7, 8, (rows, K)).astype(np.int8)
    qg = q.reshape(rows, K // 64, 64)
    qg[:, :, 3] = 7
    sc = F.bf16_round(np.exp(rng.uniform(-6, 2, (rows, K // 64))).astype(np.float32))
    v = (qg.astype(np.float32) * sc[:, :, None]).reshape(rows, K)
    got_q, got_sc = O.int4_quantize(v)
    assert np.array_equal(got_sc, sc)
    assert np.array_equal(got_q, q)


def test_int4_error_bound_and_no_minus_eight():
    rng = _rng(8)
    x = rng.standard_normal((16, 512)).astype(np.float32) * 5
    q, sc = O.int4_quantize(x)
    assert q.min() >= -7 and q.max() <= 7
    err = np.abs(x.astype(np.float64) - O.int4_dequantize(q, sc))
    bound = 0.5 * np.repeat(sc.astype(np.float64), 64, axis=1) * (1 + 2 ** -7)
    assert np.all(err <= bound)


# ------------------------------------------------------------ the layer -----

def _tiny_case(rng, M, K, N, r, bias=True):
    _, x = wl.to_bf16(rng.standard_normal((M, K)).astype(np.float32))
    _, W = wl.to_bf16(rng.standard_normal((N, K)).astype(np.float32) * 0.05)
    lam = smoothing_factors(x, W)
    _, L1 = wl.to_bf16(rng.standard_normal((K, r)).astype(np.float32) * 0.1)
    _, L2 = wl.to_bf16(rng.standard_normal((r, N)).astype(np.float32) * 0.1)
    b = wl.to_bf16(rng.standard_normal(N).astype(np.float32) * 0.1)[1] if bias else None
    return x, W, lam, L1, L2, b


@pytest.mark.parametrize("precision", ["nvfp4", "int4"])
def test_linear_matches_brute_force_triple_loop(precision):
    rng = _rng(9)
    M, K, N, r = 3, 64, 5, 4
    x, W, lam, L1, L2, b = _tiny_case(rng, M, K, N, r)
    y, y64, act, pw = O.svdq_linear(precision, x, W, lam, L1, L2, b)
    if precision == "nvfp4":
        qa = [[F.E2M1_VALUE[act["codes"][m, k]] * F.E4M3_VALUE[act["scales"][m, k // 16]] * float(act["s_a"])
               for k in range(K)] for m in range(M)]
        qw = [[F.E2M1_VALUE[pw["codes"][n, k]] * F.E4M3_VALUE[pw["scales"][n, k // 16]] * float(pw["s_w"])
               for k in range(K)] for n in range(N)]
    else:
        qa = [[float(act["q"][m, k]) * float(act["sc"][m, k // 64]) for k in range(K)] for m in range(M)]
        qw = [[float(pw["q"][n, k]) * float(pw["sc"][n, k // 64]) for k in range(K)] for n in range(N)]
    xh = act["x_hat"]
    for m in range(M):
        for n in range(N):
            acc = 0.0
            for k in range(K):
                acc += qa[m][k] * qw[n][k]
            for t in range(r):
                u = sum(float(xh[m, k]) * float(L1[k, t]) for k in range(K))
                acc += u * float(L2[t, n])
            acc += float(b[n])
            assert abs(acc - y64[m, n]) <= 1e-9 * (1 + abs(acc)), (m, n, acc, y64[m, n])


@pytest.mark.parametrize("precision", ["nvfp4", "int4"])
def test_rank_r_weight_gives_pure_lowrank_output(precision):
    rng = _rng(10)
    M, K, N, r = 8, 128, 16, 4
    L1, L2 = _dyadic_rank_r(rng, K, N, r)
    lam = np.ones(K, np.float32)
    W = (L1 @ L2).T.astype(np.float32)
    _, x = wl.to_bf16(rng.standard_normal((M, K)).astype(np.float32))
    b = wl.to_bf16(rng.standard_normal(N).astype(np.float32))[1]
    y, y64, act, pw = O.svdq_linear(precision, x, W, lam, L1, L2, b)
    want = x.astype(np.float64) @ (L1.astype(np.float64) @ L2.astype(np.float64)) + b[None, :]
    assert np.allclose(y64, want, rtol=1e-12, atol=1e-12)


def test_on_grid_operands_make_the_nvfp4_layer_exact():
    """Zero low-rank factors, power-of-two smoothing and on-grid x_hat and W_hat:
    quantization is the identity and y = x W^T + b exactly (all values dyadic)."""
    rng = _rng(11)
    M, K, N, r = 8, 128, 24, 32
    xg, _, _ = _on_grid_nvfp4(rng, M, K, np.float32(2.0 ** -8))
    wg, _, _ = _on_grid_nvfp4(rng, N, K, np.float32(2.0 ** -12))
    lam = (2.0 ** rng.integers(-2, 3, K)).astype(np.float32)
    x = (xg * lam[None, :]).astype(np.float32)
    W = (wg / lam[None, :]).astype(np.float32)
    assert np.array_equal(F.bf16_round(x), x) and np.array_equal(F.bf16_round(W), W)
    L1 = np.zeros((K, r), np.float32)
    L2 = np.zeros((r, N), np.float32)
    b = wl.to_bf16(rng.standard_normal(N).astype(np.float32))[1]
    # force the tensor scales to the powers of two used above
    pw = O.pack_weights("nvfp4", W, lam, L1, L2)
    s_w = pw["s_w"]
    pw["codes"], pw["scales"] = O.nvfp4_quantize(pw["R"], np.float32(2.0 ** -12))
    pw["s_w"] = np.float32(2.0 ** -12)
    act = O.quantize_activations("nvfp4", x, pw["inv_lam"], np.float32(2.0 ** -8))
    assert np.array_equal(act["x_hat"], xg)
    y64 = O.linear_f64("nvfp4", act, pw, L1, L2, b)
    want = x.astype(np.float64) @ W.astype(np.float64).T + b[None, :]
    assert np.allclose(y64, want, rtol=1e-12, atol=0)
    assert s_w > 0


def test_on_grid_operands_make_the_int4_layer_exact():
    rng = _rng(12)
    M, K, N, r = 4, 128, 8, 32
    def grid(rows):
        q = rng.integers(-7, 8, (rows, K)).astype(np.float32)
        q.reshape(rows, K // 64, 64)[:, :, 0] = 7
        sc = (2.0 ** rng.integers(-6, 0, (rows, K // 64))).astype(np.float32)
        return (q.reshape(rows, K // 64, 64) * sc[:, :, None]).reshape(rows, K)
    x, W = grid(M), grid(N)
    lam = np.ones(K, np.float32)
    L1 = np.zeros((K, r), np.float32)
    L2 = np.zeros((r, N), np.float32)
    y, y64, act, pw = O.svdq_linear("int4", x, W, lam, L1, L2, None)
    assert np.allclose(y64, x.astype(np.float64) @ W.astype(np.float64).T, rtol=1e-12, atol=0)


def test_quantized_layer_approximates_full_precision():
    """End-to-end sanity on the tiny workload: the W4A4 + low-rank output is a
    few percent from the unquantized x W^T (the method's purpose), and the
    low-rank branch carries most of the output."""
    inp = svdq_inputs(wl.SVDQ_CASES["tiny"])
    y, y64, act, pw = O.svdq_linear("nvfp4", inp.x, inp.W, inp.lam, inp.L1, inp.L2, inp.bias)
    ref = inp.x.astype(np.float64) @ inp.W.astype(np.float64).T
    rel = np.linalg.norm(y64 - ref) / np.linalg.norm(ref)
    assert rel < 0.08
    # without the low-rank branch, quantizing W_hat directly is much worse
    Wh = O.smooth_weight(inp.W, inp.lam).astype(np.float32)
    cw, sw = O.nvfp4_quantize(Wh, O.nvfp4_tensor_scale(Wh))
    plain = O.nvfp4_dequantize(act["codes"], act["scales"], act["s_a"]) @ \
        O.nvfp4_dequantize(cw, sw, O.nvfp4_tensor_scale(Wh)).T
    assert np.linalg.norm(plain - ref) / np.linalg.norm(ref) > rel
