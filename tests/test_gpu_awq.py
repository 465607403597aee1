"""GPU parity: the CUDA AWQ W4A16 layer against the CPU oracle, at the full
modulation-layer shape (N = 18432, K = 3072) for every token count."""
import numpy as np
import pytest
import torch

import workloads as wl
from oracle import awq as OA
from tests.helpers import assert_output_close

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,with_bias", [(1, False), (2, False), (8, False), (16, False), (5, True), (37, True)])
def test_awq_matches_oracle(M, with_bias):
    import bit_w4a4_diffusion_b200 as B
    inp = wl.make_awq_inputs(M, with_bias=with_bias)
    pk = B.awq_pack_weights(inp.W_bits)
    w = B.to_device(pk)
    x = B.bits_to_bf16(inp.x_bits, "cuda")
    bias = B.bits_to_bf16(inp.bias_bits, "cuda") if with_bias else None
    y = B.awq_w4a16_linear(x, w, bias=bias)
    torch.cuda.synchronize()
    q, sc, z = OA.awq_quantize(inp.W)
    _, y64 = OA.awq_linear(inp.x, q, sc, z, inp.bias)
    assert_output_close(y.float().cpu().numpy(), y64, f"awq M={M}")


@pytest.mark.parametrize("M,N,K", [(3, 256, 8192), (19, 512, 1024), (1, 16, 128)])
def test_awq_other_shapes(M, N, K):
    """A long K, a short one with fewer 16-row blocks than SMs, and the minimal
    shape (one 16-row block, two groups)."""
    import bit_w4a4_diffusion_b200 as B
    inp = wl.make_awq_inputs(M, N=N, K=K, seed=11, with_bias=True)
    pk = B.awq_pack_weights(inp.W_bits)
    w = B.to_device(pk)
    x = B.bits_to_bf16(inp.x_bits, "cuda")
    y = B.awq_w4a16_linear(x, w, bias=B.bits_to_bf16(inp.bias_bits, "cuda"))
    torch.cuda.synchronize()
    q, sc, z = OA.awq_quantize(inp.W)
    _, y64 = OA.awq_linear(inp.x, q, sc, z, inp.bias)
    assert_output_close(y.float().cpu().numpy(), y64, f"awq M={M} N={N} K={K}")
