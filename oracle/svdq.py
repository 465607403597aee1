"""CPU oracle for the SVDQuant ``svdq_w4a4`` linear layer (test infrastructure only).

Plain, slow, obviously correct numpy restatement of what the layer computes.
It shares no code with the CUDA library and is imported only by ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``.

What the pages say (no formula, no code is printed there):

* "Hugging Face integrates Nunchaku 4-bit diffusion inference into Diffusers",
  section "SVDQuant and the Nunchaku engine": activation outliers are moved
  into the weights, the hardest part of each weight matrix becomes a small
  16-bit low-rank branch, and the remaining residual is quantized to 4 bits;
  activations are quantized too (W4A4).
* "Nunchaku Lite" (Diffusers docs), "Supported quantization types" table:
  ``svdq_w4a4`` with ``nvfp4`` (group 16) or ``int4`` (group 64), and the
  config example there uses ``rank: 32``.

The layer computed here (the plainest reading of the pages; where they are
silent, the reading taken is stated in the docstring of the function that
takes it):

    x_hat = x * inv_lambda                  (per input channel, one fp32 multiply)
    W_hat = W * lambda                      (per input channel, exact in fp64)
    R     = fp32(W_hat - (L1 @ L2)^T)       (fp64 sum over the rank, t ascending)
    y     = bf16( Q(x_hat) @ Q(R)^T  +  x_hat @ L1 @ L2  +  b )

with Q = quantize-then-dequantize in the chosen 4-bit format.

Parity status: every function here is pinned by ``tests/test_oracle_*.py``
against format definitions, closed forms, invariants and brute force.  The
pages print no worked numbers, so nothing is pinned to the original authors'
outputs.
"""
import numpy as np

from .formats import (E2M1_VALUE, bf16_round, e2m1_encode, e4m3_decode,
                      e4m3_encode_nonneg)

NVFP4_GROUP = 16
INT4_GROUP = 64
NVFP4_TENSOR_DIVISOR = np.float32(6.0 * 448.0)   # E2M1 max times E4M3 max = 2688


# ------------------------------------------------------------ smoothing -----

def inverse_smoothing(lam):
    """inv_lambda_j = fp32(1 / lambda_j), one IEEE fp32 division."""
    lam = np.asarray(lam, dtype=np.float32)
    return (np.float32(1.0) / lam).astype(np.float32)


def smooth_activations(x, inv_lam):
    """x_hat = fp32(x) * inv_lambda, one fp32 multiply per element.

    Moving the activation outliers into the weights ("SVDQuant and the Nunchaku
    engine" section) divides input channel j by lambda_j; the division is done
    as a multiply by the stored reciprocal so that every implementation takes
    the same single rounding.
    """
    x = np.asarray(x, dtype=np.float32)
    return (x * np.asarray(inv_lam, dtype=np.float32)[None, :]).astype(np.float32)


def smooth_weight(W, lam):
    """W_hat[n, j] = W[n, j] * lambda_j in fp64 (exact: 8-bit times 24-bit mantissa)."""
    return np.asarray(W, dtype=np.float64) * np.asarray(lam, dtype=np.float32).astype(np.float64)[None, :]


def residual(W, lam, L1, L2):
    """R = fp32(W_hat - (L1 @ L2)^T), the part the 16-bit branch does not absorb.

    W is [N, K] (nn.Linear layout), L1 is [K, r], L2 is [r, N].  The rank sum
    is taken in fp64 in ascending t, one term at a time, then one subtraction
    and one rounding to fp32, so that any implementation that follows the
    same order gets the same bits (the bf16 products are exact in fp64).
    """
    W_hat = smooth_weight(W, lam)
    L1 = np.asarray(L1, dtype=np.float64)
    L2 = np.asarray(L2, dtype=np.float64)
    acc = np.zeros_like(W_hat)                     # [N, K]
    for t in range(L1.shape[1]):
        acc += L2[t, :][:, None] * L1[:, t][None, :]
    return (W_hat - acc).astype(np.float32)


# ------------------------------------------------------------ NVFP4 ---------

def nvfp4_tensor_scale(v):
    """Per-tensor fp32 scale s = amax / (6 * 448); an all-zero tensor gets s = 1."""
    amax = np.float32(np.max(np.abs(np.asarray(v, dtype=np.float32)))) if np.size(v) else np.float32(0)
    if amax == 0:
        return np.float32(1.0)
    return np.float32(amax / NVFP4_TENSOR_DIVISOR)


def nvfp4_quantize(V, s):
    """NVFP4 quantization of the rows of V along the last axis, group 16.

    Per group of 16: a = max|v|; t = fp32(a * fp32(1 / fp32(6*s)));
    sb = E4M3(t) (RNE, satfinite); d = fp32(float(sb) * s); r = fp32(1 / d);
    code = E2M1(fp32(v * r)) (RNE, satfinite, sign kept).  A group with
    d == 0 gets all-zero (+0) codes.  Every division by a scale is a multiply
    by the scale's fp32 reciprocal (one division per tensor for 6*s, one per
    block for d): the pages fix no operation order, and this is the form a
    streaming quantizer uses.

    Returns (codes uint8 [rows, K] one code per element, scales uint8 [rows, K/16]).
    """
    V = np.asarray(V, dtype=np.float32)
    rows, K = V.shape
    assert K % NVFP4_GROUP == 0
    s = np.float32(s)
    G = V.reshape(rows, K // NVFP4_GROUP, NVFP4_GROUP)
    a = np.max(np.abs(G), axis=2)                                   # exact
    six_s = np.float32(np.float32(6.0) * s)
    inv_six_s = np.float32(np.float32(1.0) / six_s)
    t = (a * inv_six_s).astype(np.float32)
    sb = e4m3_encode_nonneg(t)
    d = (e4m3_decode(sb).astype(np.float32) * s).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        r = (np.float32(1.0) / d).astype(np.float32)
        ratio = (G * r[:, :, None]).astype(np.float32)
    ratio = np.where(d[:, :, None] == 0, np.float32(0.0), ratio)
    codes = e2m1_encode(ratio)
    codes = np.where(d[:, :, None] == 0, np.uint8(0), codes).astype(np.uint8)
    return codes.reshape(rows, K), sb.astype(np.uint8)


def nvfp4_dequantize(codes, scales, s):
    """Exact fp64 value of NVFP4 data: e2m1(code) * e4m3(scale) * s."""
    codes = np.asarray(codes, dtype=np.uint8)
    rows, K = codes.shape
    val = E2M1_VALUE[codes & 0xF].reshape(rows, K // NVFP4_GROUP, NVFP4_GROUP)
    sc = e4m3_decode(scales)[:, :, None] * np.float64(np.float32(s))
    return (val * sc).reshape(rows, K)


# ------------------------------------------------------------ INT4 ----------

def int4_quantize(V):
    """Symmetric signed INT4 quantization along the last axis, group 64.

    Per group: a = max|v|; sc = bf16(a / 7) (fp32 divide, then bf16 RNE);
    r = fp32(1 / sc); q = clamp(rint(fp32(v * r)), -8, 7) with ties to even;
    q = 0 where sc == 0 (the scale applied as a reciprocal multiply, as for
    NVFP4).  Returns (q int8 [rows, K], sc float32 [rows, K/64]
    holding bf16 values).
    """
    V = np.asarray(V, dtype=np.float32)
    rows, K = V.shape
    assert K % INT4_GROUP == 0
    G = V.reshape(rows, K // INT4_GROUP, INT4_GROUP)
    a = np.max(np.abs(G), axis=2)
    sc = bf16_round((a / np.float32(7.0)).astype(np.float32))
    with np.errstate(divide="ignore", invalid="ignore"):
        r = (np.float32(1.0) / sc).astype(np.float32)
        ratio = (G * r[:, :, None]).astype(np.float32)
    q = np.rint(np.where(sc[:, :, None] == 0, np.float32(0.0), ratio))
    q = np.clip(q, -8, 7).astype(np.int8)
    return q.reshape(rows, K), sc.astype(np.float32)


def int4_dequantize(q, sc):
    q = np.asarray(q, dtype=np.int8)
    rows, K = q.shape
    G = q.astype(np.float64).reshape(rows, K // INT4_GROUP, INT4_GROUP)
    return (G * np.asarray(sc, dtype=np.float64)[:, :, None]).reshape(rows, K)


# ------------------------------------------------------------ the layer -----

def pack_weights(precision, W, lam, L1, L2):
    """Offline weight preparation: inverse smoothing, residual, weight quant.

    Returns a dict with ``inv_lam`` (fp32 [K]), ``R`` (fp32 [N, K]) and
    for "nvfp4": ``codes`` (uint8 [N, K]), ``scales`` (uint8 [N, K/16]),
    ``s_w`` (fp32); for "int4": ``q`` (int8 [N, K]), ``sc`` (fp32 [N, K/64]).
    """
    R = residual(W, lam, L1, L2)
    out = {"inv_lam": inverse_smoothing(lam), "R": R}
    if precision == "nvfp4":
        s_w = nvfp4_tensor_scale(R)
        codes, scales = nvfp4_quantize(R, s_w)
        out.update(codes=codes, scales=scales, s_w=s_w)
    elif precision == "int4":
        q, sc = int4_quantize(R)
        out.update(q=q, sc=sc)
    else:
        raise ValueError(precision)
    return out


def quantize_activations(precision, x, inv_lam, s_a=None):
    """Runtime activation side: smoothing then 4-bit quantization.

    Returns dict with ``x_hat`` and the codes/scales of the chosen format.  For
    NVFP4 the per-tensor scale ``s_a`` is a caller-supplied fp32 scalar.
    """
    x_hat = smooth_activations(x, inv_lam)
    out = {"x_hat": x_hat}
    if precision == "nvfp4":
        codes, scales = nvfp4_quantize(x_hat, s_a)
        out.update(codes=codes, scales=scales, s_a=np.float32(s_a))
    else:
        q, sc = int4_quantize(x_hat)
        out.update(q=q, sc=sc)
    return out


def lowrank_branch(x_hat, L1, L2):
    """The 16-bit branch x_hat @ L1 @ L2 in fp64 (full-precision x_hat)."""
    return (np.asarray(x_hat, dtype=np.float64) @ np.asarray(L1, dtype=np.float64)) @ \
        np.asarray(L2, dtype=np.float64)


def dequantized_act(precision, act):
    if precision == "nvfp4":
        return nvfp4_dequantize(act["codes"], act["scales"], act["s_a"])
    return int4_dequantize(act["q"], act["sc"])


def dequantized_weight(precision, pw):
    if precision == "nvfp4":
        return nvfp4_dequantize(pw["codes"], pw["scales"], pw["s_w"])
    return int4_dequantize(pw["q"], pw["sc"])


def linear_f64(precision, act, pw, L1, L2, bias):
    """y in fp64 = Q(x_hat) Q(R)^T + x_hat L1 L2 + b (before output rounding)."""
    y = dequantized_act(precision, act) @ dequantized_weight(precision, pw).T
    y += lowrank_branch(act["x_hat"], L1, L2)
    if bias is not None:
        y += np.asarray(bias, dtype=np.float64)[None, :]
    return y


def svdq_linear(precision, x, W, lam, L1, L2, bias=None, s_a=None):
    """Whole layer; returns (y as bf16 values in float32, y_f64, act, packed weights).

    ``s_a`` defaults to the NVFP4 tensor scale of x_hat (ignored for int4).
    The final bf16 rounding goes through fp32; outputs are compared within a
    tolerance, so that double rounding is immaterial.
    """
    pw = pack_weights(precision, W, lam, L1, L2)
    if precision == "nvfp4" and s_a is None:
        s_a = nvfp4_tensor_scale(smooth_activations(x, pw["inv_lam"]))
    act = quantize_activations(precision, x, pw["inv_lam"], s_a)
    y64 = linear_f64(precision, act, pw, L1, L2, bias)
    return bf16_round(y64.astype(np.float32)), y64, act, pw
