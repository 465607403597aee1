"""CPU oracle for the ``awq_w4a16`` weight-only linear layer (test infrastructure only).

"Nunchaku Lite" (Diffusers docs), "Supported quantization types" table:
``awq_w4a16 | int4 | 64`` -- an INT4 weight-only AWQ-style kernel with group
size 64.  "Hugging Face integrates Nunchaku 4-bit diffusion inference into
Diffusers", list of kernel families: it serves memory-bound,
precision-sensitive layers such as adaptive-norm modulation projections.

The pages give the format only.  Reading taken (the AWQ paper's scheme):
asymmetric uint4 with an integer zero point per group of 64 along K:

    mx = max w, mn = min w over the group
    rng = mx - mn, or |mx| for a constant group, or 1 for an all-zero group
    sc  = bf16(rng / 15)                       (fp32 divide, bf16 RNE)
    z   = clamp(rint(-mn / sc), 0, 15)         (fp32 divide, ties to even)
    q   = clamp(rint(w / sc) + z, 0, 15)
    deq = (q - z) * sc
    y   = bf16( x @ deq^T + b )

The per-input-channel AWQ activation scale is folded offline into x and W
(part of the synthetic input recipe), so the layer sees plain bf16 x and W.
"""
import numpy as np

from .formats import bf16_round

AWQ_GROUP = 64


def awq_quantize(W):
    """Returns (q uint8 [N, K] in 0..15, sc float32 [N, K/64] (bf16 values), z uint8 [N, K/64])."""
    W = np.asarray(W, dtype=np.float32)
    N, K = W.shape
    assert K % AWQ_GROUP == 0
    G = W.reshape(N, K // AWQ_GROUP, AWQ_GROUP)
    mx = G.max(axis=2)
    mn = G.min(axis=2)
    rng = (mx - mn).astype(np.float32)
    rng = np.where(rng == 0, np.abs(mx), rng)
    rng = np.where(rng == 0, np.float32(1.0), rng).astype(np.float32)
    sc = bf16_round((rng / np.float32(15.0)).astype(np.float32))
    z = np.clip(np.rint((-mn / sc).astype(np.float32)), 0, 15)
    q = np.clip(np.rint((G / sc[:, :, None]).astype(np.float32)) + z[:, :, None], 0, 15)
    return q.astype(np.uint8).reshape(N, K), sc.astype(np.float32), z.astype(np.uint8)


def awq_dequantize(q, sc, z):
    q = np.asarray(q, dtype=np.float64)
    N, K = q.shape
    G = q.reshape(N, K // AWQ_GROUP, AWQ_GROUP)
    deq = (G - np.asarray(z, dtype=np.float64)[:, :, None]) * np.asarray(sc, dtype=np.float64)[:, :, None]
    return deq.reshape(N, K)


def awq_linear(x, q, sc, z, bias=None):
    """Returns (y as bf16 values in float32, y in fp64)."""
    y = np.asarray(x, dtype=np.float64) @ awq_dequantize(q, sc, z).T
    if bias is not None:
        y += np.asarray(bias, dtype=np.float64)[None, :]
    return bf16_round(y.astype(np.float32)), y
