"""svdq_w4a4_linear_noalloc through the C ABI, against svdq_w4a4_linear.

The no-allocation entry point serves callers that cannot allocate device
memory while they run the layer (graph capture on a stream they do not own,
plugins that receive only input and output pointers, allocators closed after
start-up).  It keeps the quantized activations in the library's built-in
device scratch instead of a caller workspace.  This file is collected last
so that a run stopping at the first failure has run every other test.
"""
import numpy as np
import pytest
import torch

import workloads as wl
from tests.helpers import assert_output_close, svdq_inputs

pytestmark = pytest.mark.gpu


def _layer(name, **kw):
    import bit_w4a4_diffusion_b200 as B
    c = wl.scaled_case(wl.SVDQ_CASES[name], **kw)
    inp = svdq_inputs(c)
    pk = B.svdq_pack_weights("nvfp4", inp.W_bits, inp.lam, inp.L1_bits, inp.L2_bits)
    w = B.to_device(pk)
    x = B.bits_to_bf16(inp.x_bits, "cuda")
    bias = B.bits_to_bf16(inp.bias_bits, "cuda") if inp.bias_bits is not None else None
    return B, c, inp, w, x, bias


def test_noalloc_matches_workspace_entry_point_twice():
    # Two calls in a row with different shapes and inputs: the second call
    # reuses the scratch the first one left behind.
    for name, kw in [("qkv", dict(M=300, N=1024)), ("mlp_up", dict(M=129, N=512, K=2048))]:
        B, c, inp, w, x, bias = _layer(name, **kw)
        y_ref = B.svdq_w4a4_linear("nvfp4", x, w, float(inp.act_scale), bias=bias)
        y_na = B.svdq_w4a4_linear_noalloc("nvfp4", x, w, float(inp.act_scale), bias=bias)
        torch.cuda.synchronize()
        assert_output_close(y_na.float().cpu().numpy(), y_ref.float().cpu().numpy().astype(np.float64),
                            f"noalloc vs workspace ({c.name})")


def test_noalloc_rejects_shapes_beyond_the_scratch():
    import bit_w4a4_diffusion_b200 as B
    cap = B.lib.svdq_noalloc_scratch_bytes()
    assert cap == 32 * 2 ** 20
    M, K = 8192, 12288                         # needs about 58 MB of scratch
    assert B.workspace_bytes("nvfp4", M, K) > cap
    x = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
    w = {"N": 256, "K": K, "rank": 32, "weight_scale_f": 1.0,
         **{k: torch.empty(16, dtype=torch.uint8, device="cuda")
            for k in ("inv_smooth", "lora_down", "codes", "scales", "lora_up")}}
    with pytest.raises(B.SvdqError) as e:
        B.svdq_w4a4_linear_noalloc("nvfp4", x, w, 1.0)
    assert e.value.status == 2 and "scratch" in str(e.value)
