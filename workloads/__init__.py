"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module holds no step of the method: it draws random tensors (x, W,
bias, the Gaussian test matrix of the low-rank calibration, rotary tables)
and hands x and W to a caller-supplied calibration function that returns the
layer's remaining inputs (smoothing factors, the rank-r factors and the
static activation scale): the tests pass the oracle's, the benchmark the
library's own ``svdq_calibrate``.  For the AWQ layer it folds the
per-input-channel scale s_j = mean_i(|x_ij|)^0.5 into W diag(s) and x / s
(both rounded to bf16), which shapes the inputs without entering the
layer's arithmetic.

The pages' own workloads (ERNIE-Image-Turbo and Flux Schnell weights and
prompts) are not available; these shapes and distributions stand in for
them: diffusion-transformer projections over 4096 tokens (a 64x64 latent
patch grid) with hidden size 3072.

Every random number comes from numpy's PCG64 seeded with the case's seed.
Tensors are drawn in fp32 and rounded to bf16 (round-to-nearest-even).
"""
from dataclasses import dataclass, field

import numpy as np
import torch

# --------------------------------------------------------------- helpers ----


def to_bf16(a):
    """fp32 array -> (uint16 bf16 bit patterns, float32 values of those bf16)."""
    t = torch.from_numpy(np.ascontiguousarray(np.asarray(a, dtype=np.float32))).to(torch.bfloat16)
    bits = t.view(torch.int16).numpy().view(np.uint16).copy()
    return bits, t.to(torch.float32).numpy().copy()


def _rng(seed):
    return np.random.Generator(np.random.PCG64(seed))


def outlier_activations(rng, M, K, n_outlier, factor, gelu=False):
    """x ~ N(0,1) (optionally GELU(N(0,1)), exact erf form), then n_outlier
    channels chosen without replacement multiplied by ``factor``."""
    x = rng.standard_normal((M, K), dtype=np.float32)
    if gelu:
        xt = torch.from_numpy(x.astype(np.float64))
        x = (0.5 * xt * (1.0 + torch.erf(xt / np.sqrt(2.0)))).numpy().astype(np.float32)
    if n_outlier:
        ch = rng.choice(K, n_outlier, replace=False)
        x[:, ch] *= np.float32(factor)
    return x


def gaussian_weight(rng, N, K, std, n_outlier_entries=0, factor=1.0):
    W = rng.standard_normal((N, K), dtype=np.float32) * np.float32(std)
    if n_outlier_entries:
        idx = rng.choice(N * K, n_outlier_entries, replace=False)
        W.reshape(-1)[idx] *= np.float32(factor)
    return W


OVERSAMPLE = 8       # columns of the calibration test matrix beyond the rank


def calibration_test_matrix(case):
    """The Gaussian test matrix [N, rank + OVERSAMPLE] (fp64) of the case's
    low-rank calibration, from its own seeded stream."""
    return _rng([*np.atleast_1d(_seed(case.seed)), 7]).standard_normal((case.N, case.rank + OVERSAMPLE))


# --------------------------------------------------------------- cases ------


@dataclass
class SvdqCase:
    name: str
    precision: str             # "nvfp4" | "int4"
    M: int
    K: int
    N: int
    rank: int
    seed: object
    n_outlier_ch: int
    outlier_factor: float
    w_outlier_entries: int = 0
    w_outlier_factor: float = 1.0
    bias_std: float = 0.0
    gelu: bool = False
    w_std: float = 0.02

    def flops(self):
        return 2.0 * self.M * self.N * self.K


@dataclass
class SvdqInputs:
    case: SvdqCase
    x_bits: np.ndarray          # uint16 [M, K]
    x: np.ndarray               # float32 values of x_bits
    W_bits: np.ndarray          # uint16 [N, K]
    W: np.ndarray
    lam: np.ndarray             # float32 [K]
    L1_bits: np.ndarray         # uint16 [K, r]
    L1: np.ndarray
    L2_bits: np.ndarray         # uint16 [r, N]
    L2: np.ndarray
    bias_bits: object = None    # uint16 [N] or None
    bias: object = None
    act_scale: float = 1.0      # calibrated NVFP4 activation tensor scale (fp32)
    extra: dict = field(default_factory=dict)


def _seed(seed):
    return list(seed) if isinstance(seed, (tuple, list)) else seed


def make_svdq_inputs(case: SvdqCase, calibrate) -> SvdqInputs:
    """Draw x, W, bias for ``case``; ``calibrate(x_bits, W_bits, omega, rank)``
    returns (lambda fp32 [K], L1 bf16 bits [K, r], L2 bf16 bits [r, N], s_a)."""
    rng = _rng(_seed(case.seed))
    x = outlier_activations(rng, case.M, case.K, case.n_outlier_ch, case.outlier_factor, case.gelu)
    W = gaussian_weight(rng, case.N, case.K, case.w_std, case.w_outlier_entries, case.w_outlier_factor)
    bias = None
    if case.bias_std > 0:
        bias = rng.standard_normal(case.N, dtype=np.float32) * np.float32(case.bias_std)
    x_bits, x_v = to_bf16(x)
    W_bits, W_v = to_bf16(W)
    lam, L1_bits, L2_bits, s_a = calibrate(x_bits, W_bits, calibration_test_matrix(case), case.rank)
    lam = np.asarray(lam, dtype=np.float32)
    L1_bits = np.ascontiguousarray(L1_bits, dtype=np.uint16)
    L2_bits = np.ascontiguousarray(L2_bits, dtype=np.uint16)
    L1_v = (L1_bits.astype(np.uint32) << 16).view(np.float32)
    L2_v = (L2_bits.astype(np.uint32) << 16).view(np.float32)
    b_bits = b_v = None
    if bias is not None:
        b_bits, b_v = to_bf16(bias)
    return SvdqInputs(case, x_bits, x_v, W_bits, W_v, lam, L1_bits, L1_v, L2_bits, L2_v, b_bits, b_v,
                      np.float32(s_a))


# The five workloads (diffusion-transformer shapes).  "1% of channels" is
# round(0.01 * K); "0.1% of entries" is round(0.001 * N * K).
SVDQ_CASES = {
    "tiny": SvdqCase("tiny", "nvfp4", 256, 1024, 1024, 32, 0, 8, 40.0),
    "qkv": SvdqCase("qkv", "nvfp4", 4096, 3072, 9216, 32, 1, 31, 50.0,
                    w_outlier_entries=28312, w_outlier_factor=10.0, bias_std=0.01),
    "mlp_up": SvdqCase("mlp_up", "nvfp4", 4096, 3072, 12288, 32, 2, 31, 50.0),
    "mlp_down": SvdqCase("mlp_down", "nvfp4", 4096, 12288, 3072, 32, (2, 1), 123, 50.0, gelu=True),
}
for _m in (1024, 2048, 4096, 8192):
    SVDQ_CASES[f"int4_m{_m}"] = SvdqCase(f"int4_m{_m}", "int4", _m, 3072, 3072, 32, 3, 31, 50.0)


def scaled_case(case: SvdqCase, M=None, N=None, K=None, name=None):
    """The same recipe at a reduced size (for cases the oracle finishes in seconds)."""
    M = case.M if M is None else M
    N = case.N if N is None else N
    K = case.K if K is None else K
    n_ch = max(1, round(case.n_outlier_ch * K / case.K)) if case.n_outlier_ch else 0
    n_w = round(case.w_outlier_entries * (N * K) / (case.N * case.K))
    return SvdqCase(name or f"{case.name}_{M}x{K}x{N}", case.precision, M, K, N, case.rank,
                    case.seed, n_ch, case.outlier_factor, n_w, case.w_outlier_factor,
                    case.bias_std, case.gelu, case.w_std)


@dataclass
class AwqInputs:
    M: int
    N: int
    K: int
    x_bits: np.ndarray
    x: np.ndarray
    W_bits: np.ndarray
    W: np.ndarray
    bias_bits: object = None
    bias: object = None


def make_awq_inputs(M, N=18432, K=3072, seed=4, with_bias=False):
    """Modulation-linear workload: x ~ N(0,1) [M, K], W ~ N(0, 0.02) [N, K],
    with the AWQ per-input-channel scale s_j = mean_i(|x_ij|)^0.5 folded in
    (W diag(s), x / s), then both rounded to bf16.  Bias zero unless asked."""
    rng = _rng(seed)
    x = rng.standard_normal((M, K), dtype=np.float32)
    W = gaussian_weight(rng, N, K, 0.02)
    s = np.sqrt(np.mean(np.abs(x), axis=0)).astype(np.float32)
    s[s == 0] = 1.0
    x = (x / s[None, :]).astype(np.float32)
    W = (W * s[None, :]).astype(np.float32)
    bias = rng.standard_normal(N, dtype=np.float32) * np.float32(0.01) if with_bias else None
    xb, xv = to_bf16(x)
    Wb, Wv = to_bf16(W)
    bb = bv = None
    if bias is not None:
        bb, bv = to_bf16(bias)
    return AwqInputs(M, N, K, xb, xv, Wb, Wv, bb, bv)


AWQ_MS = (1, 2, 8, 16)


def make_rope_norm_inputs(M, heads, seed=5, head_dim=128, base=10000.0):
    """Per-feature RMSNorm weights for Q and K heads (uniform in [0.5, 1.5])
    and rotary tables of tokens 0..M-1: angle(m, i) = m * base^(-2i/head_dim),
    as fp32 cos / sin [M, head_dim/2]."""
    g = _rng(seed)
    gamma_q = g.uniform(0.5, 1.5, head_dim).astype(np.float32)
    gamma_k = g.uniform(0.5, 1.5, head_dim).astype(np.float32)
    i = np.arange(head_dim // 2, dtype=np.float64)
    ang = np.arange(M, dtype=np.float64)[:, None] * base ** (-2.0 * i[None, :] / head_dim)
    return gamma_q, gamma_k, np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)

