"""Number-format codecs for the CPU oracle (test infrastructure only).

This module, like the rest of ``oracle/``, is a plain, slow, obviously
correct restatement used to check the CUDA library.  Only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
import it; the product path never does.

Formats (the pages name them, they do not define them; the definitions are
the public OCP Microscaling (MX) v1.0 element formats and NVIDIA's NVFP4
description):

* E2M1 ("nvfp4" element, Nunchaku Lite docs, "Supported quantization types"
  table: ``svdq_w4a4 | nvfp4 | 16``): 1 sign bit, 2 exponent bits (bias 1),
  1 mantissa bit, no inf/NaN.  Magnitudes for codes 0..7 are
  0, 0.5, 1, 1.5, 2, 3, 4, 6; bit 3 is the sign.
* E4M3 ("fn" variant, used unsigned as the per-16 group scale): 4 exponent
  bits (bias 7), 3 mantissa bits, no inf, 0x7F/0xFF are NaN, max 448,
  smallest subnormal 2^-9.
* bf16: the top half of an IEEE binary32.

Encoders are written as the definition of round-to-nearest with ties to the
even code over the finite grid, saturating to the largest finite value
("satfinite"): for each input the two grid neighbours are found and the
nearer one taken; on an exact tie the neighbour with the even code wins.
"""
import numpy as np
import torch

# ---------------------------------------------------------------- decoders --

def e2m1_magnitude(code):
    """Magnitude of a 3-bit E2M1 code (no sign) from the format fields."""
    code = int(code)
    e, m = (code >> 1) & 0x3, code & 0x1
    if e == 0:
        return 0.5 * m                      # subnormal: m * 2^(1-bias) * 2^-1
    return 2.0 ** (e - 1) * (1.0 + 0.5 * m)


def e4m3_value(byte):
    """Value of an E4M3 byte (fn variant) from the format fields; NaN for 0x7F/0xFF."""
    byte = int(byte)
    s = -1.0 if byte & 0x80 else 1.0
    e, m = (byte >> 3) & 0xF, byte & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return s * (m / 8.0) * 2.0 ** -6
    return s * 2.0 ** (e - 7) * (1.0 + m / 8.0)


E2M1_MAG = np.array([e2m1_magnitude(c) for c in range(8)], dtype=np.float64)
E2M1_VALUE = np.array([(-1.0 if c & 8 else 1.0) * E2M1_MAG[c & 7] for c in range(16)],
                      dtype=np.float64)
E4M3_VALUE = np.array([e4m3_value(b) for b in range(256)], dtype=np.float64)
E4M3_MAX = 448.0
E2M1_MAX = 6.0


def e2m1_decode(codes):
    """Signed value of 4-bit E2M1 codes (uint8 array with one code per element)."""
    return E2M1_VALUE[np.asarray(codes, dtype=np.uint8) & 0xF]


def e4m3_decode(bytes_):
    return E4M3_VALUE[np.asarray(bytes_, dtype=np.uint8)]


# ---------------------------------------------------------------- encoders --

def _nearest_code(mag, grid, codes):
    """Round non-negative magnitudes to the nearest grid value, ties to even code.

    ``grid`` is ascending with ``codes`` its (consecutive) codes.  Values above
    the last grid point saturate to it.  All comparisons are exact in fp64
    because every grid value and every fp32 input is exactly representable.
    """
    mag = np.asarray(mag, dtype=np.float64)
    hi = np.searchsorted(grid, mag, side="left")          # grid[hi] >= mag
    hi = np.minimum(hi, len(grid) - 1)
    lo = np.maximum(hi - 1, 0)
    d_lo = mag - grid[lo]
    d_hi = grid[hi] - mag
    take_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (codes[hi] % 2 == 0))
    out = np.where(take_hi, codes[hi], codes[lo])
    out = np.where(mag >= grid[-1], codes[-1], out)         # satfinite
    out = np.where(mag <= grid[0], codes[0], out)
    return out.astype(np.uint8)


_E2M1_CODES = np.arange(8, dtype=np.int64)
_E4M3_POS_CODES = np.arange(127, dtype=np.int64)            # 0x00..0x7E (0x7F is NaN)
_E4M3_POS_GRID = E4M3_VALUE[:127].copy()


def e2m1_encode(v):
    """fp32 -> 4-bit E2M1 code, round-to-nearest-even, satfinite, sign kept.

    The sign bit is the sign of the input, so a negative value that rounds to
    zero gives code 0x8 (IEEE-style signed zero).
    """
    v = np.asarray(v, dtype=np.float32)
    mag_code = _nearest_code(np.abs(v).astype(np.float64), E2M1_MAG, _E2M1_CODES)
    sign = np.signbit(v).astype(np.uint8) << 3
    return (mag_code | sign).astype(np.uint8)


def e4m3_encode_nonneg(t):
    """Non-negative fp32 -> E4M3 byte, round-to-nearest-even, satfinite (max 448)."""
    t = np.asarray(t, dtype=np.float32)
    if np.any(t < 0) or np.any(np.isnan(t)):
        raise ValueError("e4m3_encode_nonneg expects finite non-negative inputs")
    return _nearest_code(t.astype(np.float64), _E4M3_POS_GRID, _E4M3_POS_CODES)


def bf16_round(x):
    """fp32 -> nearest bf16 (ties to even), returned as float32 values.

    Uses torch's CPU cast as the rounding primitive.
    """
    t = torch.from_numpy(np.ascontiguousarray(np.asarray(x, dtype=np.float32)))
    return t.to(torch.bfloat16).to(torch.float32).numpy()


def bf16_bits(x):
    """fp32 -> bf16 bit patterns (uint16), round-to-nearest-even."""
    t = torch.from_numpy(np.ascontiguousarray(np.asarray(x, dtype=np.float32)))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def bf16_from_bits(bits):
    """bf16 bit patterns (uint16) -> float32 values (exact)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32)
