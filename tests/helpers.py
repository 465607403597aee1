"""Shared test utilities: output tolerance, nibble unpacking, sampling."""
import numpy as np

REL_L2_TOL = 5e-3        # relative L2 error bound on the layer output
MAX_ABS_TOL = 2e-2       # max-abs error bound, in units of rms(y)


def nibbles(packed):
    """[rows, K/2] bytes -> [rows, K] codes (element 2j = low nibble)."""
    packed = np.asarray(packed, dtype=np.uint8)
    return np.stack([packed & 0xF, packed >> 4], axis=-1).reshape(packed.shape[0], -1)


def bf16_half_ulp(v):
    """Half a bf16 unit in the last place at |v| (the output format's own rounding)."""
    a = np.abs(np.asarray(v, dtype=np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return 0.5 * 2.0 ** (e - 7)


def output_errors(y_gpu, y_ref):
    """(relative L2 error, max over elements of (|d| - half-ulp(y_ref)) / rms(y_ref))."""
    y_gpu = np.asarray(y_gpu, dtype=np.float64)
    y_ref = np.asarray(y_ref, dtype=np.float64)
    d = y_gpu - y_ref
    rel = np.linalg.norm(d) / max(np.linalg.norm(y_ref), 1e-300)
    rms = np.sqrt(np.mean(y_ref ** 2))
    excess = np.max(np.abs(d) - bf16_half_ulp(y_ref)) / max(rms, 1e-300)
    return rel, excess


def assert_output_close(y_gpu, y_ref, what=""):
    """The layer's output bound: relative L2 <= 5e-3 and, per element,
    |y - y_ref| <= 2e-2 rms(y_ref) + half a bf16 ulp of y_ref, where y_ref is
    the oracle's output before its final bf16 rounding."""
    rel, excess = output_errors(y_gpu, y_ref)
    assert np.all(np.isfinite(y_gpu)), f"{what}: non-finite outputs"
    assert rel <= REL_L2_TOL, f"{what}: relative L2 error {rel:.3e} > {REL_L2_TOL}"
    assert excess <= MAX_ABS_TOL, f"{what}: max-abs excess {excess:.3e} rms > {MAX_ABS_TOL}"
    return rel, excess
