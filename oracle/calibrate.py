"""CPU oracle for the offline calibration that produces an svdq_w4a4 layer's
inputs (test infrastructure only: imported by ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``).

Page: "Hugging Face integrates Nunchaku 4-bit diffusion inference into
Diffusers", section "SVDQuant and the Nunchaku engine": activation outliers
are migrated into the weights, then the hardest part of each weight matrix
is absorbed by a 16-bit low-rank branch obtained by decomposing it; the
"Nunchaku Lite" docs' config example uses rank 32.  The pages give no
formula; the reading taken here, where each choice is this module's own:

    lambda_j   = sqrt(max_i |x_ij| / max_n |W_nj|) in fp32, 1 where a max is 0
                 (migration strength 1/2 over the calibration batch x)
    A          = (W diag(lambda))^T in fp64, [K, N]
    L1, L2     = rank-r factors of A from randomized subspace iteration
                 (Halko, Martinsson & Tropp, "Finding structure with
                 randomness", 2011, Algorithm 4.4) with the given Gaussian test
                 matrix Omega [N, r + p] and q power iterations:
                   Q = qr(A Omega); q times: Z = qr(A^T Q), Q = qr(A Z);
                   B = Q^T A = Ub S Vt (SVD); U = Q Ub[:, :r];
                 each column of U negated if its largest-magnitude entry is
                 negative (the first one on a tie), the row of Vt with it;
                 L1 = bf16(U_r S_r) [K, r], L2 = bf16(Vt_r) [r, N]
    s_a        = max |x_ij * fp32(1 / lambda_j)| / 2688 in fp32 (1 if 0): the
                 static NVFP4 activation tensor scale of the calibration batch

The test matrix is an input (drawn by the caller), so that every
implementation runs the same iteration.

Parity status: pinned by ``tests/test_oracle_calibrate.py``.
"""
import numpy as np

from .formats import bf16_bits


def smoothing_factors(x, W):
    """lambda_j = sqrt(max_i|x_ij| / max_n|W_nj|) in fp32; 1 where a max is 0."""
    ax = np.max(np.abs(np.asarray(x, dtype=np.float32)), axis=0).astype(np.float32)
    aw = np.max(np.abs(np.asarray(W, dtype=np.float32)), axis=0).astype(np.float32)
    ok = (ax > 0) & (aw > 0)
    lam = np.ones_like(ax)
    lam[ok] = np.sqrt((ax[ok] / aw[ok]).astype(np.float32)).astype(np.float32)
    return lam.astype(np.float32)


def lowrank_factors(A, r, omega, power_iters=4):
    """Rank-r factors (L1 = U_r S_r [K, r], L2 = Vt_r [r, N], fp64) of A
    [K, N] by randomized subspace iteration with test matrix omega [N, l]."""
    A = np.asarray(A, dtype=np.float64)
    Q, _ = np.linalg.qr(A @ np.asarray(omega, dtype=np.float64))
    for _ in range(power_iters):
        Z, _ = np.linalg.qr(A.T @ Q)
        Q, _ = np.linalg.qr(A @ Z)
    B = Q.T @ A
    Ub, S, Vt = np.linalg.svd(B, full_matrices=False)
    U = Q @ Ub[:, :r]
    S = S[:r]
    Vt = Vt[:r].copy()
    sign = np.sign(U[np.argmax(np.abs(U), axis=0), np.arange(r)])
    sign[sign == 0] = 1.0
    U *= sign[None, :]
    Vt *= sign[:, None]
    return U * S[None, :], Vt


def act_scale(x, lam):
    """max_ij |x_ij * fp32(1/lambda_j)| / 2688 in fp32 (1 for an all-zero batch)."""
    inv = (np.float32(1.0) / np.asarray(lam, dtype=np.float32)).astype(np.float32)
    amax = np.float32(np.max(np.abs((np.asarray(x, dtype=np.float32) * inv[None, :]).astype(np.float32))))
    return np.float32(amax / np.float32(2688.0)) if amax > 0 else np.float32(1.0)


def calibrate(x_bits, W_bits, omega, rank, power_iters=4):
    """The whole recipe on bf16 bit patterns: x [M, K], W [N, K].

    Returns (lambda fp32 [K], L1 bf16 bits [K, r], L2 bf16 bits [r, N],
    s_a fp32)."""
    x = (np.asarray(x_bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)
    W = (np.asarray(W_bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)
    lam = smoothing_factors(x, W)
    A = (W.astype(np.float64) * lam.astype(np.float64)[None, :]).T
    L1, L2 = lowrank_factors(A, rank, omega, power_iters)
    return lam, bf16_bits(L1.astype(np.float32)), bf16_bits(L2.astype(np.float32)), act_scale(x, lam)
