"""The arithmetic the INT4 layer's fp16 operands rest on, checked on the CPU
over every case ("Nunchaku Lite" docs, "Supported quantization types":
int4 with one bf16 scale per 64 elements).

A row is scaled by 2^-E with E = floor(log2 of the row's largest scale) - 12,
clamped to [-100, 100].  The claim: for every bf16 scale s of the row with
s >= 2^(E - 17) (every group within 2^29 of the largest) and every code q in
[-8, 7], s 2^-E q is exactly an fp16 value, and the largest magnitude (8
times the largest scale) stays within fp16's 65504.  A bf16 significand has
8 bits and a code at most 3, so the product has at most 11, fp16's
precision; its last bit is at least 2^(e_s - 7 - E), which fp16 (smallest
subnormal step 2^-24) holds exactly when e_s >= E - 17.

Checked for every E in [-100, 100], every bf16 significand and every
exponent from E - 17 up to the largest the row can hold; the step just
below the window is shown not to be exact for some code, so the bound is
the tightest one.  The claim holds while E is not clamped, i.e. for rows
whose largest scale lies in [2^-88, 2^113): at the top the clamped E = 100
leaves 8 times a scale of 2^113 or more beyond fp16's range, and at the
bottom the window stays at 2^-117, narrower than 2^29 below the largest."""
import numpy as np
import pytest

CODES = np.arange(-8, 8, dtype=np.float64)
SIGNIFICANDS = 1.0 + np.arange(128, dtype=np.float64) / 128.0     # all bf16 significands in [1, 2)


def _exact_in_fp16(v):
    v = np.asarray(v, dtype=np.float64)
    return np.all(v.astype(np.float16).astype(np.float64) == v)


def _row_exponent(max_scale):
    """E from the row's largest scale (positive), as the layer defines it."""
    _, ex = np.frexp(max_scale)          # max_scale = m 2^ex, m in [0.5, 1)
    return int(np.clip(ex - 1 - 12, -100, 100))


@pytest.mark.parametrize("E", range(-100, 101, 1))
def test_every_scale_in_the_window_is_exact(E):
    # Largest scales whose row exponent is E without the clamp:
    # [2^(E + 12), 2^(E + 13)).
    top = np.ldexp(SIGNIFICANDS, E + 12)
    assert all(_row_exponent(s) == E for s in top[[0, -1]])
    # fp16's largest finite value bounds the row's largest product.
    assert np.max(np.abs(np.ldexp(top, -E)[:, None] * CODES[None, :])) <= 65504
    # Every scale from 2^(E - 17) up to the largest: exact for every code.
    exps = np.arange(E - 17, E + 13)
    s = np.ldexp(SIGNIFICANDS[None, :], exps[:, None]).ravel()
    v = np.ldexp(s, -E)[:, None] * CODES[None, :]
    assert _exact_in_fp16(v)


def test_the_window_is_tight():
    E = 0
    below = np.ldexp(SIGNIFICANDS, E - 18)          # one exponent under the window
    v = np.ldexp(below, -E)[:, None] * CODES[None, :]
    assert not _exact_in_fp16(v)
    # Only the odd-significand products lose their last bit there.
    odd = np.ldexp(1.0 + 1.0 / 128.0, E - 18)
    assert not _exact_in_fp16([np.ldexp(odd, -E)])


def test_row_exponent_edges():
    # A bf16 scale just under a power of two and the power of two itself.
    assert _row_exponent(np.float64(1.0)) == -12
    assert _row_exponent(np.float64(2.0 - 1.0 / 128.0)) == -12
    assert _row_exponent(np.float64(2.0)) == -11
    # The clamp: tiny and huge scales.
    assert _row_exponent(np.ldexp(1.0, -120)) == -100
    assert _row_exponent(np.ldexp(1.0, 120)) == 100


def test_clamped_rows():
    """Outside [2^-88, 2^113) the clamp changes the picture (the layer's
    documented domain ends there)."""
    # Top: the largest scale 2^113 gets E = 100, and 8 s 2^-100 = 2^16 is not
    # a finite fp16 value; just under 2^113 the row is still fine.
    assert _row_exponent(np.ldexp(1.0, 113)) == 100
    with np.errstate(over="ignore"):
        assert not np.isfinite(np.float16(np.ldexp(np.ldexp(1.0, 113), -100) * 8))
    assert _row_exponent(np.ldexp(SIGNIFICANDS[-1], 112)) == 100
    assert _exact_in_fp16(np.ldexp(SIGNIFICANDS[-1], 112 - 100) * CODES)
    # Bottom: the largest scale 2^-100 gets E = -100; a group 2^-20 below it
    # (within 2^29) but under 2^-117 is not exact for every significand.
    assert _row_exponent(np.ldexp(1.0, -100)) == -100
    v = np.ldexp(np.ldexp(SIGNIFICANDS, -120), 100)[:, None] * CODES[None, :]
    assert not _exact_in_fp16(v)
    # At the window's edge it is.
    v = np.ldexp(np.ldexp(SIGNIFICANDS, -117), 100)[:, None] * CODES[None, :]
    assert _exact_in_fp16(v)
