"""Pins for the operation order inside the oracle's 4-bit quantizers (CPU only).

The pages fix the formats ("Nunchaku Lite" docs, "Supported quantization
types" table: nvfp4 with an E4M3 scale per 16, int4 with a scale per 64) but
not how a value is divided by its scale.  The oracle reads it as a multiply
by the scale's fp32 reciprocal, the form of NVIDIA's two-level NVFP4 scaling
(its 2025 NVFP4 pretraining report multiplies each value by a per-block
encode scale, the reciprocal of the block's decode scale) and of any
streaming quantizer, which computes one reciprocal per block:

    NVFP4:  sb = E4M3(a * fl(1 / fl(6 s))),  code = E2M1(v * fl(1 / fl(E4M3(sb) s)))
    INT4:   q  = rint(v * fl(1 / sc)),        sc = bf16(a / 7)

Two kinds of pins, with different jobs:

* The order itself: inputs where the reciprocal form and a plain division
  give different codes or scale bytes (tests/quant_order_cases.py finds
  them).  The oracle must give the reciprocal form's result on every one of
  them, and there must be enough of them that a switch to division cannot
  go unnoticed.
* Everything but the order, against the exact arithmetic: on random data,
  each scale byte and code must be the round-to-nearest-even of the EXACT
  quotient (fp64; the operands are fp32 and the grids are dyadic), except
  where that quotient lies within the fp32 rounding of the reciprocal form
  (a few units of 2^-24, relative) of a rounding midpoint -- there either
  neighbour is allowed.  A dropped term, a wrong scale, a wrong factor of 6
  or a biased rounding fails this regardless of the order.
"""
import numpy as np
import pytest

from oracle import formats as F
from oracle import svdq as O
from tests import quant_order_cases as QC

# Per-tensor scales whose reciprocals are inexact in fp32.
S_VALUES = [np.float32(0.0123457), np.float32(3.1e-5), np.float32(7.77)]


@pytest.mark.parametrize("s", S_VALUES)
def test_nvfp4_oracle_takes_the_reciprocal_form(s):
    rows, where = QC.nvfp4_rows(s)
    kinds = [w[2] for w in where]
    assert kinds.count("code") >= 24 and kinds.count("scale") >= 24, "too few order cases found"
    codes, sb = O.nvfp4_quantize(rows, s)
    for r, j, kind, c in where:
        if kind == "code":
            a, v, sb_case, c_rec, c_div = c
            assert sb[r, j] == sb_case
            assert codes[r, 16 * j + 1] == c_rec and c_rec != c_div, (a, v)
        else:
            a, sb_rec, sb_div = c
            assert sb[r, j] == sb_rec and sb_rec != sb_div, a


def test_int4_oracle_takes_the_reciprocal_form():
    rows, where = QC.int4_rows(32)
    assert len(where) >= 24, "too few order cases found"
    q, sc = O.int4_quantize(rows)
    for r, j, (a, v, sc_case, q_rec, q_div) in where:
        assert sc[r, j] == sc_case
        assert q[r, 64 * j + 1] == q_rec and q_rec != q_div, (a, v)


# ------------------------------------------------------- exact-quotient bound

def _nearest_even(x, grid, rel):
    """Nearest point of the ascending, dyadic `grid` to x >= 0 (fp64), ties
    to the even index, saturating at the ends; also the two neighbours and
    whether x lies within rel * x of their midpoint."""
    x = np.minimum(np.asarray(x, dtype=np.float64), grid[-1])
    hi = np.minimum(np.searchsorted(grid, x, side="left"), len(grid) - 1)
    lo = np.maximum(hi - 1, 0)
    on_grid = grid[hi] == x
    lo = np.where(on_grid, hi, lo)
    mid = (grid[lo] + grid[hi]) / 2
    tie = np.where(lo % 2 == 0, lo, hi)
    idx = np.where(x < mid, lo, np.where(x > mid, hi, tie))
    ambiguous = (lo != hi) & (np.abs(x - mid) <= rel * x)
    return idx, lo, hi, ambiguous


# The reciprocal form's deviation from the exact quotient: rounding of the
# reciprocal, of the product and (NVFP4) of d = E4M3 * s, each <= 2^-24.
REL = 4 * 2.0 ** -24


def _random_rows(seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((64, 1024)).astype(np.float32)
    x *= np.exp(rng.uniform(-6, 6, (64, 1))).astype(np.float32)      # many magnitudes
    x[:, rng.choice(1024, 12, replace=False)] *= 50                    # outlier channels
    return x


@pytest.mark.parametrize("seed", [11, 12])
def test_nvfp4_within_rounding_of_the_exact_quotient(seed):
    x = _random_rows(seed)
    s = O.nvfp4_tensor_scale(x)
    codes, sb = O.nvfp4_quantize(x, s)
    G = x.reshape(64, 64, 16).astype(np.float64)
    a = np.max(np.abs(G), axis=2)
    s64 = np.float64(s)
    # scale bytes: E4M3 round-to-nearest-even of a / (6 s), exact in fp64 up to 2^-53
    e4m3_grid = F.E4M3_VALUE[:127]
    idx, lo, hi, amb = _nearest_even(a / (6.0 * s64), e4m3_grid, REL)
    sb = sb.astype(np.int64)
    assert np.all((sb == idx) | (amb & ((sb == lo) | (sb == hi))))
    assert np.mean(amb) < 1e-3
    # codes: E2M1 round-to-nearest-even of v / (E4M3(sb) s), sign kept
    d = F.E4M3_VALUE[sb] * s64                        # exact product of a 4-bit and a 24-bit significand
    cg = codes.reshape(64, 64, 16)
    # a scale that underflows to 0 gives an all-(+0) group
    zero = d == 0
    assert np.any(zero) and np.all(cg[zero] == 0)
    live = ~zero
    ratio = G[live] / d[live][:, None]
    cidx, clo, chi, camb = _nearest_even(np.abs(ratio), F.E2M1_MAG, REL)
    mag = cg[live] & 7
    sign = cg[live] >> 3
    assert np.all((mag == cidx) | (camb & ((mag == clo) | (mag == chi))))
    assert np.all(sign == np.signbit(G[live]).astype(np.uint8))
    assert np.mean(camb) < 1e-3


@pytest.mark.parametrize("seed", [13, 14])
def test_int4_within_rounding_of_the_exact_quotient(seed):
    x = _random_rows(seed)
    q, sc = O.int4_quantize(x)
    G = x.reshape(64, 16, 64).astype(np.float64)
    a = np.max(np.abs(G), axis=2)
    # the scale: a / 7 rounded to bf16 (a single rounding of the fp32 quotient)
    assert np.all(np.abs(sc - a / 7.0) <= 2.0 ** -8 * a / 7.0 + 2.0 ** -24 * a / 7.0)
    ratio = G / sc.astype(np.float64)[:, :, None]
    near = np.rint(ratio)
    frac = np.abs(ratio - np.trunc(ratio))
    amb = np.abs(frac - 0.5) <= REL * np.abs(ratio)
    qg = q.reshape(64, 16, 64).astype(np.float64)
    lower, upper = np.floor(ratio), np.ceil(ratio)
    ok = (qg == np.clip(near, -8, 7)) | (amb & ((qg == lower) | (qg == upper)))
    assert np.all(ok)
    assert np.mean(amb) < 1e-3
