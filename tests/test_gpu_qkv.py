"""GPU parity of the fused QKV projection with RMSNorm and RoPE against the
CPU oracle: the layer's output before rounding goes through the oracle's
normalization and rotation in fp64, and the CUDA result must satisfy the
layer's output bound (``helpers.assert_output_close``)."""
import numpy as np
import pytest
import torch

import workloads as wl
from oracle import qkv as OQ
from oracle import svdq as O
from tests.helpers import assert_output_close, svdq_inputs

pytestmark = pytest.mark.gpu


def _lib():
    import bit_w4a4_diffusion_b200 as B
    return B


def _setup(M, K, heads):
    B = _lib()
    c = wl.scaled_case(wl.SVDQ_CASES["qkv"], M=M, K=K, N=3 * heads * 128)
    inp = svdq_inputs(c)
    pk = B.svdq_pack_weights("nvfp4", inp.W_bits, inp.lam, inp.L1_bits, inp.L2_bits)
    gq, gk, cos, sin = wl.make_rope_norm_inputs(M, heads)
    # the library takes the rotary tables pair-major: [64, M]
    dev = {k: torch.from_numpy(np.ascontiguousarray(v)).cuda()
           for k, v in (("gq", gq), ("gk", gk), ("cos", cos.T), ("sin", sin.T))}
    return inp, pk, B.to_device(pk), (gq, gk, cos, sin), dev


def _ref(inp, rows, gq, gk, cos, sin, heads):
    ref_pw = O.pack_weights("nvfp4", inp.W, inp.lam, inp.L1, inp.L2)
    act = O.quantize_activations("nvfp4", inp.x[rows], ref_pw["inv_lam"], np.float32(inp.act_scale))
    return OQ.qkv_layer_f64(act, ref_pw, inp.L1, inp.L2, inp.bias, gq, gk, cos[rows], sin[rows], heads)


@pytest.mark.parametrize("M,K,heads", [
    (300, 1024, 2),     # ragged M
    (129, 256, 1),      # N = 384: the last tile is half a tile (one head)
    (1, 512, 3),        # a single token, 4.5 tiles
    (512, 768, 4),
])
@pytest.mark.parametrize("kernel", ["pair", "single"])
def test_qkv_norm_rope_matches_oracle(M, K, heads, kernel, monkeypatch):
    """Both NVFP4 GEMM kernels carry the epilogue (the CTA-pair one by
    default)."""
    monkeypatch.setenv("SVDQ_NVFP4_GEMM_KERNEL", kernel)
    B = _lib()
    inp, pk, w, (gq, gk, cos, sin), d = _setup(M, K, heads)
    x = B.bits_to_bf16(inp.x_bits, "cuda")
    bias = B.bits_to_bf16(inp.bias_bits, "cuda") if inp.bias_bits is not None else None
    s_a = float(inp.act_scale)
    codes, scales, lora = B.svdq_quantize_act("nvfp4", x, w["inv_smooth"], w["lora_down"], s_a, w["weight_scale_f"])
    alpha = float(np.float32(np.float32(s_a) * np.float32(pk["weight_scale"][0])))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = B.svdq_w4a4_gemm_qkv_norm_rope(codes, scales, lora, w, alpha, heads, d["gq"], d["gk"], d["cos"], d["sin"],
                                       bias=bias, dev_status=status)
    y2 = B.svdq_w4a4_qkv_norm_rope_linear(x, w, s_a, heads, d["gq"], d["gk"], d["cos"], d["sin"], bias=bias)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref = _ref(inp, np.arange(M), gq, gk, cos, sin, heads)
    assert_output_close(y.float().cpu().numpy(), ref, f"qkv {M}x{K} heads={heads}")
    assert torch.equal(y, y2), "the one-call layer differs from quantize + GEMM"


def test_qkv_norm_rope_full_size_sampled():
    """The DiT QKV projection: 4096 tokens, 3072 -> 9216 (24 heads)."""
    B = _lib()
    M, K, heads = 4096, 3072, 24
    inp, pk, w, (gq, gk, cos, sin), d = _setup(M, K, heads)
    x = B.bits_to_bf16(inp.x_bits, "cuda")
    bias = B.bits_to_bf16(inp.bias_bits, "cuda") if inp.bias_bits is not None else None
    y = B.svdq_w4a4_qkv_norm_rope_linear(x, w, float(inp.act_scale), heads, d["gq"], d["gk"], d["cos"], d["sin"],
                                         bias=bias)
    torch.cuda.synchronize()
    rows = np.array([0, 1, 127, 128, 1000, 2047, 2048, 3001, 4094, 4095])
    ref = _ref(inp, rows, gq, gk, cos, sin, heads)
    assert_output_close(y.float().cpu().numpy()[rows], ref, "qkv full size (sampled rows)")


def test_qkv_rejects_bad_head_layout():
    B = _lib()
    inp, pk, w, _, d = _setup(64, 256, 1)
    x = B.bits_to_bf16(inp.x_bits, "cuda")
    with pytest.raises(B.SvdqError):
        B.svdq_w4a4_qkv_norm_rope_linear(x, w, 1.0, 2, d["gq"], d["gk"], d["cos"], d["sin"])   # N != 3*2*128
