"""Pins for the oracle's number-format codecs (CPU only).

Each codec is checked against something other than itself: the OCP format
tables (golden files), torch's independent float8 cast, a bit-level bf16
rounding written from IEEE 754, and brute-force nearest-value search.
"""
import math
import os

import numpy as np
import pytest
import torch

from oracle import formats as F

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_table(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            a, b = line.split()
            rows.append((a, b))
    return rows


def test_e2m1_decode_matches_ocp_table():
    for code, val in _read_table("e2m1_table.txt"):
        got = F.e2m1_decode(np.array([int(code)], dtype=np.uint8))[0]
        want = float(val)
        assert got == want and math.copysign(1, got) == math.copysign(1, want), (code, got, want)


def test_e4m3_decode_matches_ocp_points():
    for byte, val in _read_table("e4m3_points.txt"):
        got = F.e4m3_decode(np.array([int(byte, 16)], dtype=np.uint8))[0]
        if val == "nan":
            assert np.isnan(got)
        else:
            assert got == float(val), (byte, got, val)


def test_e4m3_decode_matches_torch_float8_for_all_bytes():
    raw = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = raw.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = F.E4M3_VALUE
    both_nan = np.isnan(ref) & np.isnan(got)
    assert np.all(both_nan | (ref == got))


def test_e2m1_encode_ties_and_saturation():
    for val, code in _read_table("rne_ties.txt"):
        got = int(F.e2m1_encode(np.array([float(val)], dtype=np.float32))[0])
        assert got == int(code), (val, got, code)


def _brute_nearest_even(mag, grid):
    """Index of the nearest grid value, ties to the even index, by full scan."""
    best, best_d = None, None
    for i, g in enumerate(grid):
        d = abs(mag - g)
        if best is None or d < best_d or (d == best_d and i % 2 == 0):
            best, best_d = i, d
    return best


def test_e2m1_encode_brute_force_sweep():
    rng = np.random.default_rng(11)
    v = np.concatenate([
        rng.uniform(-7, 7, 4000).astype(np.float32),
        np.arange(-6.5, 6.5, 0.125, dtype=np.float32),     # every midpoint and grid point
        np.array([0.0, -0.0, 1e-30, -1e-30, 6.0001, -6.0001], dtype=np.float32),
    ])
    codes = F.e2m1_encode(v)
    for x, c in zip(v, codes):
        mag = min(abs(float(x)), 6.0)
        want = _brute_nearest_even(mag, list(F.E2M1_MAG))
        assert (int(c) & 7) == want, (x, c, want)
        assert (int(c) >> 3) == int(np.signbit(x)), (x, c)


def test_e4m3_encode_matches_torch_cast_in_range():
    rng = np.random.default_rng(12)
    t = np.concatenate([
        np.exp(rng.uniform(np.log(1e-4), np.log(448.0), 20000)).astype(np.float32),
        F.E4M3_VALUE[:127].astype(np.float32),                              # grid points
        ((F.E4M3_VALUE[:126] + F.E4M3_VALUE[1:127]) / 2).astype(np.float32),  # midpoints
        np.array([0.0, 2.0 ** -10, 2.0 ** -11, 1e-30], dtype=np.float32),
    ])
    got = F.e4m3_encode_nonneg(t)
    ref = torch.from_numpy(t).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(got, ref)


def test_e4m3_encode_saturates():
    t = np.array([448.0, 460.0, 464.0, 1e6, 3.4e38], dtype=np.float32)
    assert np.all(F.e4m3_encode_nonneg(t) == 0x7E)


def _bf16_rne_bits(x):
    """IEEE 754 roundTiesToEven of binary32 to its top 16 bits (finite inputs)."""
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lower = u & 0xFFFF
    upper = u >> 16
    round_up = (lower > 0x8000) | ((lower == 0x8000) & ((upper & 1) == 1))
    return (upper + round_up).astype(np.uint16)


def test_bf16_round_matches_ieee_bit_rounding():
    rng = np.random.default_rng(13)
    x = np.concatenate([rng.standard_normal(50000).astype(np.float32) * 100,
                        np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -1.0 - 2 ** -8, 0.0, -0.0],
                                 dtype=np.float32)])
    assert np.array_equal(F.bf16_bits(x), _bf16_rne_bits(x))
    assert np.array_equal(F.bf16_round(x).view(np.uint32) >> 16, _bf16_rne_bits(x).astype(np.uint32))
    assert np.array_equal(F.bf16_from_bits(_bf16_rne_bits(x)), F.bf16_round(x))
