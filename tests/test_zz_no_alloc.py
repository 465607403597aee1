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
from oracle import svdq as O
from tests.helpers import assert_output_close, svdq_inputs

pytestmark = pytest.mark.gpu


def _layer(name, prec="nvfp4", **kw):
    import bit_w4a4_diffusion_b200 as B
    c = wl.scaled_case(wl.SVDQ_CASES[name], **kw)
    inp = svdq_inputs(c)
    pk = B.svdq_pack_weights(prec, inp.W_bits, inp.lam, inp.L1_bits, inp.L2_bits)
    w = B.to_device(pk)
    x = B.bits_to_bf16(inp.x_bits, "cuda")
    bias = B.bits_to_bf16(inp.bias_bits, "cuda") if inp.bias_bits is not None else None
    return B, c, inp, w, x, bias


CALLS = [("nvfp4", "qkv", dict(M=300, N=1024)),
         ("nvfp4", "mlp_up", dict(M=129, N=512, K=2048)),
         ("int4", "int4_m1024", dict(M=200, N=512, K=1024))]


def test_noalloc_matches_workspace_entry_point_twice():
    # Calls in a row with different precisions, shapes and inputs: each call
    # reuses the scratch the one before it left behind.  Both entry points run
    # the same deterministic kernels on the same inputs, so the outputs must
    # be identical bit for bit; the oracle bound is checked as well.
    for prec, name, kw in CALLS:
        B, c, inp, w, x, bias = _layer(name, prec, **kw)
        s_a = float(inp.act_scale) if prec == "nvfp4" else 1.0
        y_ref = B.svdq_w4a4_linear(prec, x, w, s_a, bias=bias)
        y_na = B.svdq_w4a4_linear_noalloc(prec, x, w, s_a, bias=bias)
        torch.cuda.synchronize()
        assert torch.equal(y_na, y_ref), f"noalloc differs from the workspace entry point ({prec}, {c.name})"
        ref_pw = O.pack_weights(prec, inp.W, inp.lam, inp.L1, inp.L2)
        act = O.quantize_activations(prec, inp.x, ref_pw["inv_lam"], np.float32(s_a))
        y64 = O.linear_f64(prec, act, ref_pw, inp.L1, inp.L2, inp.bias)
        assert_output_close(y_na.float().cpu().numpy(), y64, f"noalloc vs oracle ({prec}, {c.name})")


def test_noalloc_rejects_shapes_beyond_the_scratch():
    import bit_w4a4_diffusion_b200 as B
    cap = B.lib.svdq_noalloc_scratch_bytes()
    assert cap == 32 * 2 ** 20
    M, K = 8192, 12288                         # needs about 58 MB of scratch
    assert B.workspace_bytes("nvfp4", M, 256, K) > cap
    x = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
    w = {"N": 256, "K": K, "rank": 32, "weight_scale_f": 1.0,
         **{k: torch.empty(16, dtype=torch.uint8, device="cuda")
            for k in ("inv_smooth", "lora_down", "codes", "scales", "lora_up")}}
    with pytest.raises(B.SvdqError) as e:
        B.svdq_w4a4_linear_noalloc("nvfp4", x, w, 1.0)
    assert e.value.status == 2 and "scratch" in str(e.value)
