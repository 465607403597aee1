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


def check_nvfp4_near_boundary(v_ref, s, codes, scales, delta):
    """NVFP4 codes and scales decided from values that carry an error.

    v_ref [rows, K] (fp64) is the exact input of the quantizer and ``delta``
    (broadcastable to v_ref) bounds the error of the values the device
    quantized.  Each group's scale must be the E4M3 rounding of
    max|v| / (6 s) for some max|v| within delta of the exact one, and each
    code, decided with the device's own scale, the E2M1 rounding of some
    value within delta of the exact one (both encoders are monotone, so the
    allowed results are the range between the roundings of v - delta and
    v + delta).  Returns the fraction of codes that differ from the
    quantizer applied to v_ref itself.
    """
    from oracle import formats as F
    from oracle import svdq as O
    v_ref = np.asarray(v_ref, dtype=np.float64)
    rows, K = v_ref.shape
    delta = np.broadcast_to(np.asarray(delta, dtype=np.float64), v_ref.shape)
    s32 = np.float32(s)
    inv6s = np.float32(np.float32(1.0) / np.float32(np.float32(6.0) * s32))
    G = v_ref.reshape(rows, K // 16, 16)
    D = delta.reshape(rows, K // 16, 16)
    a = np.max(np.abs(G), axis=2)
    da = np.max(D, axis=2)
    lo_sb = F.e4m3_encode_nonneg((np.maximum(a - da, 0) * float(inv6s)).astype(np.float32))
    hi_sb = F.e4m3_encode_nonneg(((a + da) * float(inv6s)).astype(np.float32))
    assert np.all((scales >= lo_sb) & (scales <= hi_sb)), "a group scale is off by more than the value error"
    d = (F.e4m3_decode(scales).astype(np.float32) * s32).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        r = np.where(d > 0, (np.float32(1.0) / d).astype(np.float32), np.float32(0)).astype(np.float64)
    vals = F.E2M1_VALUE[np.asarray(codes) & 0xF].reshape(rows, K // 16, 16)
    lo = F.E2M1_VALUE[F.e2m1_encode(((G - D) * r[:, :, None]).astype(np.float32))]
    hi = F.E2M1_VALUE[F.e2m1_encode(((G + D) * r[:, :, None]).astype(np.float32))]
    ok = (vals >= lo - 1e-12) & (vals <= hi + 1e-12)
    assert np.all(ok), f"{np.sum(~ok)} codes are off by more than the value error"
    ref_codes, _ = O.nvfp4_quantize(v_ref.astype(np.float32), s32)
    return float(np.mean(ref_codes != np.asarray(codes)))


def identical_decision_rows(got_codes, got_scales, ref_codes, ref_scales):
    """Rows whose NVFP4 codes [rows, K] and scale bytes [rows, K/16] equal
    the reference's everywhere (boolean mask)."""
    same_c = np.all(np.asarray(got_codes) == np.asarray(ref_codes), axis=1)
    same_s = np.all(np.asarray(got_scales) == np.asarray(ref_scales), axis=1)
    return same_c & same_s


def svdq_inputs(case):
    """The seeded inputs of `case`, calibrated by the oracle (smoothing,
    rank-r factors, activation scale)."""
    import workloads as wl
    from oracle import calibrate as OC
    return wl.make_svdq_inputs(case, OC.calibrate)
