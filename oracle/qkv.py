"""CPU oracle for the fused QKV projection with RMSNorm and RoPE (test
infrastructure only: imported by ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py``, never by the product path).

Page: "Nunchaku Lite" (Diffusers docs), section "Fused kernels": the original
Nunchaku engine combines the Q, K and V projections with RMSNorm and RoPE
(its table credits the fusion with 1.27x per step); Nunchaku Lite runs the
same layers without it.  The pages give neither a formula nor the head
layout.  The reading taken here is the one of diffusion transformers with
query/key normalization:

    v        = the QKV layer's output before rounding, [M, 3 H d], columns
               [Q | K | V], head h of each part in columns [h d, (h + 1) d)
    n(u)     = u / sqrt(mean(u^2) + eps) * gamma       over the d features of
               one head (RMSNorm, gamma_q for Q, gamma_k for K, eps = 1e-6)
    rope(u)  = for each pair (u[2i], u[2i + 1]) of a head, i < d/2, rotated by
               the angle of token m and pair i:
               (a, b) -> (a cos - b sin, a sin + b cos)
    out      = [rope(n(Q)) | rope(n(K)) | V]

cos and sin are caller-supplied [M, d/2] tables (the positions and
frequencies are the model's business).

Parity status: pinned by ``tests/test_oracle_qkv.py`` (unit RMS, scale
invariance, rotation identities and composition, and a brute-force loop with
Python's complex arithmetic).
"""
import numpy as np

from . import svdq as O

HEAD_DIM = 128
RMS_EPS = 1e-6


def rmsnorm(u, gamma, eps=RMS_EPS):
    """RMSNorm over the last axis of u [..., d] in fp64, times gamma [d]."""
    u = np.asarray(u, dtype=np.float64)
    ms = np.mean(u * u, axis=-1, keepdims=True)
    return u / np.sqrt(ms + eps) * np.asarray(gamma, dtype=np.float64)


def rope(u, cos, sin):
    """Rotate the pairs (u[..., 2i], u[..., 2i + 1]) of u [M, ..., d] by the
    angle whose cosine and sine are cos[m, i], sin[m, i] ([M, d/2])."""
    u = np.asarray(u, dtype=np.float64)
    a, b = u[..., 0::2], u[..., 1::2]
    shape = (u.shape[0],) + (1,) * (u.ndim - 2) + (u.shape[-1] // 2,)
    c = np.asarray(cos, dtype=np.float64).reshape(shape)
    s = np.asarray(sin, dtype=np.float64).reshape(shape)
    out = np.empty_like(u)
    out[..., 0::2] = a * c - b * s
    out[..., 1::2] = a * s + b * c
    return out


def qkv_norm_rope(v, gamma_q, gamma_k, cos, sin, heads, d=HEAD_DIM, eps=RMS_EPS):
    """[rope(n(Q)) | rope(n(K)) | V] of v [M, 3 heads d] (fp64)."""
    v = np.asarray(v, dtype=np.float64)
    M = v.shape[0]
    hd = heads * d
    assert v.shape[1] == 3 * hd
    q = v[:, :hd].reshape(M, heads, d)
    k = v[:, hd:2 * hd].reshape(M, heads, d)
    out = v.copy()
    out[:, :hd] = rope(rmsnorm(q, gamma_q, eps), cos, sin).reshape(M, hd)
    out[:, hd:2 * hd] = rope(rmsnorm(k, gamma_k, eps), cos, sin).reshape(M, hd)
    return out


def qkv_layer_f64(act, pw, L1, L2, bias, gamma_q, gamma_k, cos, sin, heads, d=HEAD_DIM, eps=RMS_EPS):
    """The fused layer in fp64: the svdq_w4a4 NVFP4 layer's output before
    rounding, then the normalization and rotation above."""
    v = O.linear_f64("nvfp4", act, pw, L1, L2, bias)
    return qkv_norm_rope(v, gamma_q, gamma_k, cos, sin, heads, d, eps)
