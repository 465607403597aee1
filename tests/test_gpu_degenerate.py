"""GPU parity on the method's degenerate cases ("Hugging Face integrates
Nunchaku 4-bit diffusion inference into Diffusers", section "SVDQuant and the
Nunchaku engine": the low-rank branch absorbs part of the weight, the 4-bit
residual carries the rest).

- An all-zero activation: every code, scale and low-rank value is zero, so
  y is the bias, bit for bit, in both precisions and through every INT4
  GEMM option of the layer.
- A weight that is exactly rank r after smoothing: the residual R is zero,
  so every weight code is zero and the layer's output is the low-rank
  branch alone, x_hat L1 L2 + b, which the oracle evaluates in fp64.
"""
import numpy as np
import pytest
import torch

import workloads as wl
from oracle import svdq as O
from tests.helpers import assert_output_close, nibbles

pytestmark = pytest.mark.gpu

M, N, K, R = 200, 384, 512, 32


def _bias(rng):
    return wl.to_bf16(rng.standard_normal(N, dtype=np.float32) * np.float32(0.01))


def _exact_rank_inputs(seed):
    """lambda = 1, L1 and L2 small integers times 2^-4, and W = (L1 L2)^T,
    whose entries are integers times 2^-8 of magnitude at most 2^-1: exact
    in bf16, so R = W diag(lambda) - (L1 L2)^T is exactly zero."""
    rng = np.random.default_rng(seed)
    L1 = rng.integers(-2, 3, size=(K, R)).astype(np.float32) * np.float32(2.0 ** -4)
    L2 = rng.integers(-2, 3, size=(R, N)).astype(np.float32) * np.float32(2.0 ** -4)
    W = (L1.astype(np.float64) @ L2.astype(np.float64)).T.astype(np.float32)
    L1_bits, L1v = wl.to_bf16(L1)
    L2_bits, L2v = wl.to_bf16(L2)
    W_bits, Wv = wl.to_bf16(W)
    assert np.array_equal(L1v, L1) and np.array_equal(L2v, L2) and np.array_equal(Wv, W)
    x_bits, xv = wl.to_bf16(rng.standard_normal((M, K), dtype=np.float32))
    b_bits, bv = _bias(rng)
    return x_bits, xv, W_bits, Wv, L1_bits, L1v, L2_bits, L2v, b_bits, bv


@pytest.mark.parametrize("prec,option", [("nvfp4", None), ("int4", None), ("int4", "dq"), ("int4", "i8")])
def test_zero_activation_gives_the_bias(prec, option, monkeypatch):
    import bit_w4a4_diffusion_b200 as B
    if option is not None:
        monkeypatch.setenv("SVDQ_INT4_LAYER_GEMM", option)
    c = wl.scaled_case(wl.SVDQ_CASES["tiny"], M=M, N=N, K=K)
    inp = wl.make_svdq_inputs(c, B.svdq_calibrate)
    pk = B.svdq_pack_weights(prec, inp.W_bits, inp.lam, inp.L1_bits, inp.L2_bits)
    w = B.to_device(pk)
    b_bits, _ = _bias(np.random.default_rng(5))
    bias = B.bits_to_bf16(b_bits, "cuda")
    x = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    y = B.svdq_w4a4_linear(prec, x, w, 1.0, bias=bias)
    codes, scales, lora = B.svdq_quantize_act(prec, x, w["inv_smooth"], w["lora_down"], 1.0, w["weight_scale_f"])
    torch.cuda.synchronize()
    assert not codes.any() and not scales.any() and not lora.float().any()
    assert torch.equal(y, bias.expand(M, N)), "y is not the bias"


@pytest.mark.parametrize("prec", ["nvfp4", "int4"])
def test_exact_rank_weight_gives_the_low_rank_branch(prec):
    import bit_w4a4_diffusion_b200 as B
    x_bits, xv, W_bits, Wv, L1_bits, L1v, L2_bits, L2v, b_bits, bv = _exact_rank_inputs(11)
    lam = np.ones(K, np.float32)
    pk = B.svdq_pack_weights(prec, W_bits, lam, L1_bits, L2_bits)
    assert not np.any(pk["codes"]), "the residual of an exactly rank-r weight must quantize to zero codes"
    w = B.to_device(pk)
    x = B.bits_to_bf16(x_bits, "cuda")
    bias = B.bits_to_bf16(b_bits, "cuda")
    s_a = float(np.float32(np.max(np.abs(xv)) / np.float32(2688.0)))
    y = B.svdq_w4a4_linear(prec, x, w, s_a, bias=bias)
    torch.cuda.synchronize()
    ref_pw = O.pack_weights(prec, Wv, lam, L1v, L2v)
    assert not np.any(ref_pw["codes"] if prec == "nvfp4" else ref_pw["q"])
    act = O.quantize_activations(prec, xv, ref_pw["inv_lam"], np.float32(s_a) if prec == "nvfp4" else None)
    y64 = O.linear_f64(prec, act, ref_pw, L1v, L2v, bv)
    # The oracle's value is the low-rank branch plus the bias.
    lowrank = (xv.astype(np.float64) @ L1v.astype(np.float64)) @ L2v.astype(np.float64) + bv.astype(np.float64)
    assert np.allclose(y64, lowrank, rtol=0, atol=1e-12 * np.abs(lowrank).max())
    assert_output_close(y.float().cpu().numpy(), y64, f"exact rank-{R} weight ({prec})")
    # The codes of x are the oracle's.
    codes, _, _ = B.svdq_quantize_act(prec, x, w["inv_smooth"], w["lora_down"], s_a, w["weight_scale_f"])
    torch.cuda.synchronize()
    if prec == "nvfp4":
        assert np.array_equal(nibbles(codes.cpu().numpy()), act["codes"])
