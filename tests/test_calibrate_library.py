"""The library's host calibration (svdq_calibrate, C++) against the oracle:
the same randomized subspace iteration with the same test matrix, so the
smoothing factors and the activation scale agree bit for bit and the bf16
low-rank factors agree to the last bit but for rounding-boundary cases."""
import numpy as np
import pytest

import bit_w4a4_diffusion_b200 as B
import workloads as wl
from oracle import calibrate as OC


def _draw(c):
    rng = wl._rng(c.seed if not isinstance(c.seed, tuple) else list(c.seed))
    x = wl.outlier_activations(rng, c.M, c.K, c.n_outlier_ch, c.outlier_factor, c.gelu)
    W = wl.gaussian_weight(rng, c.N, c.K, c.w_std, c.w_outlier_entries, c.w_outlier_factor)
    return wl.to_bf16(x)[0], wl.to_bf16(W)[0], wl.calibration_test_matrix(c)


def _vals(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


@pytest.mark.parametrize("name,kw", [
    ("tiny", {}),
    ("qkv", dict(M=64, N=1024, K=512)),
    ("mlp_up", dict(M=128, N=768, K=1024)),
    ("mlp_down", dict(M=96, N=512, K=1536)),
    ("int4_m1024", dict(M=64, N=512, K=768)),
])
def test_library_calibration_matches_oracle(name, kw):
    c = wl.SVDQ_CASES[name]
    if kw:
        c = wl.scaled_case(c, **kw)
    xb, Wb, om = _draw(c)
    lam, L1, L2, s_a = B.svdq_calibrate(xb, Wb, om, c.rank)
    lam_o, L1_o, L2_o, s_o = OC.calibrate(xb, Wb, om, c.rank)
    assert np.array_equal(lam, lam_o)
    assert s_a == s_o
    assert np.mean(_vals(L1) == _vals(L1_o)) >= 0.999 and np.mean(_vals(L2) == _vals(L2_o)) >= 0.999
    P, Po = _vals(L1) @ _vals(L2), _vals(L1_o) @ _vals(L2_o)
    assert np.linalg.norm(P - Po) <= 1e-3 * np.linalg.norm(Po)


def test_library_calibration_edge_cases():
    rng = np.random.default_rng(44)
    M, N, K, r = 8, 64, 48, 4
    x = rng.standard_normal((M, K)).astype(np.float32)
    W = rng.standard_normal((N, K)).astype(np.float32) * 0.1
    x[:, 3] = 0.0          # a silent input channel
    W[:, 5] = 0.0          # an all-zero weight column
    xb, Wb = wl.to_bf16(x)[0], wl.to_bf16(W)[0]
    om = rng.standard_normal((N, r + 8))
    lam, L1, L2, s_a = B.svdq_calibrate(xb, Wb, om, r)
    lam_o, L1_o, L2_o, s_o = OC.calibrate(xb, Wb, om, r)
    assert lam[3] == 1.0 and lam[5] == 1.0 and np.array_equal(lam, lam_o) and s_a == s_o
    # The zero weight column gives a row of L1 that is zero up to rounding
    # noise (about 1e-17), which the two implementations round differently.
    a, b = _vals(L1), _vals(L1_o)
    tiny = np.maximum(np.abs(a), np.abs(b)) < 1e-12 * np.abs(b).max()
    assert np.all(tiny[5]) and np.array_equal(a[~tiny], b[~tiny])
    assert np.array_equal(_vals(L2), _vals(L2_o))
    with pytest.raises(B.SvdqError):
        B.svdq_calibrate(xb, Wb, rng.standard_normal((N, 60)), r)     # rank + oversample > K
