"""CPU oracle for the GELU-MLP fusion of two svdq_w4a4 layers (test
infrastructure only: imported by ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py``, never by the product path).

Page: "Nunchaku Lite" (Diffusers docs), section "Fused kernels": the original
Nunchaku engine runs the MLP with a fused GELU kernel (its table credits the
"GELU-MLP fusion" with 1.06x per step); Nunchaku Lite runs the same layers
without it.  The pages give no formula.  The reading taken here (the
plainest composition of the two layers that never stores the up output):

    v     = up layer output before its bf16 rounding
          = Q(x_hat) Q(R_up)^T + x_hat L1_up L2_up + b_up        (fp64 here)
    h     = GELU(v) = v * Phi(v) = 0.5 v (1 + erf(v / sqrt 2))  (exact erf form)
    h_hat = h * inv_lambda_down                                  (down layer's smoothing)
    codes, scales = NVFP4(h_hat, s_down)                         (down layer's activation quantizer)
    u     = h_hat L1_down,   lora_act = u / (s_down * s_w_down)
    y     = down layer's 4-bit GEMM on (codes, scales, lora_act) + b_down

that is, the unfused pipeline "up layer -> GELU -> down layer" with the up
layer's output kept at full precision instead of being rounded to bf16 and
re-read: the fused kernel never stores it.  The exact-erf GELU is the form
used for the synthetic down-projection activations of this build's MLP
workload; the pages name no form.

Parity status: pinned by ``tests/test_oracle_mlp.py`` (standard normal table
values, the odd-part identity, the location of GELU's minimum, closed-form
compositions and a brute-force loop over a tiny MLP).
"""
import numpy as np
from scipy.special import erf

from . import svdq as O


def gelu(v):
    """GELU(v) = 0.5 v (1 + erf(v / sqrt(2))) in fp64 (v times the standard
    normal CDF)."""
    v = np.asarray(v, dtype=np.float64)
    return 0.5 * v * (1.0 + erf(v / np.sqrt(2.0)))


def up_output_f64(act_up, pw_up, L1_up, L2_up, bias_up):
    """v: the up layer's output in fp64, before any rounding."""
    return O.linear_f64("nvfp4", act_up, pw_up, L1_up, L2_up, bias_up)


def gelu_requantize(v, inv_lam_down, s_down):
    """GELU, the down layer's smoothing and its NVFP4 activation quantizer.

    Returns a dict in the shape of ``svdq.quantize_activations``: ``x_hat``
    (fp64 h_hat), ``codes``, ``scales`` (the quantizer applied to
    fp32(h_hat), the precision in which the fused kernel decides them) and
    ``s_a`` = s_down.
    """
    h_hat = gelu(v) * np.asarray(inv_lam_down, dtype=np.float32).astype(np.float64)[None, :]
    codes, scales = O.nvfp4_quantize(h_hat.astype(np.float32), s_down)
    return {"x_hat": h_hat, "codes": codes, "scales": scales, "s_a": np.float32(s_down)}


def lora_act(h_hat, L1_down, s_down, s_w_down):
    """u / (s_down * s_w_down) with u = h_hat L1_down in fp64: the value the
    down layer's GEMM expects in its low-rank slot (its alpha divided out)."""
    alpha = np.float64(np.float32(np.float32(s_down) * np.float32(s_w_down)))
    return (np.asarray(h_hat, dtype=np.float64) @ np.asarray(L1_down, dtype=np.float64)) / alpha


def mlp_f64(act_up, pw_up, L1_up, L2_up, bias_up, pw_down, L1_down, L2_down, bias_down, s_down):
    """The whole fused MLP in fp64: returns (y_down before rounding, the
    down layer's activation dict, v)."""
    v = up_output_f64(act_up, pw_up, L1_up, L2_up, bias_up)
    act_d = gelu_requantize(v, pw_down["inv_lam"], s_down)
    y = O.linear_f64("nvfp4", act_d, pw_down, L1_down, L2_down, bias_down)
    return y, act_d, v
