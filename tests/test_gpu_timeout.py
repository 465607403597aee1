"""Failure detection without a GPU fault: every mbarrier wait in the NVFP4,
INT4, GELU-MLP and QKV GEMM kernels is bounded by the library's wait limit.  With
the limit set to 1 ns the first wait that is not already satisfied gives up;
the kernel must report a timeout code through dev_status, drain its own
copies and MMAs, free its tensor memory and return, leaving the context
usable: the next call with the normal limit gives the correct result."""
import numpy as np
import pytest
import torch

import workloads as wl
from oracle import svdq as O
from tests.helpers import assert_output_close, svdq_inputs

pytestmark = pytest.mark.gpu

TIMEOUT_CODES = (1, 2, 3, 4)   # producer, MMA, epilogue, drain (csrc/svdq_internal.h)


@pytest.mark.parametrize("kernel", ["single", "pair"])
def test_gemm_wait_timeout_reports_and_recovers(kernel, monkeypatch):
    import bit_w4a4_diffusion_b200 as B
    monkeypatch.setenv("SVDQ_NVFP4_GEMM_KERNEL", kernel)
    c = wl.scaled_case(wl.SVDQ_CASES["qkv"], M=640, N=2048)   # several tiles per CTA
    inp = svdq_inputs(c)
    pk = B.svdq_pack_weights("nvfp4", inp.W_bits, inp.lam, inp.L1_bits, inp.L2_bits)
    w = B.to_device(pk)
    bias = B.bits_to_bf16(inp.bias_bits, "cuda") if inp.bias_bits is not None else None
    x = B.bits_to_bf16(inp.x_bits, "cuda")
    s_a = float(inp.act_scale)
    codes, scales, lora = B.svdq_quantize_act("nvfp4", x, w["inv_smooth"], w["lora_down"], s_a, w["weight_scale_f"])
    alpha = float(np.float32(np.float32(s_a) * np.float32(pk["weight_scale"][0])))
    torch.cuda.synchronize()

    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    old = B.get_timeout_ns()
    try:
        B.set_timeout_ns(1)
        B.svdq_w4a4_gemm("nvfp4", codes, scales, lora, w, alpha, bias=bias, dev_status=status)
        torch.cuda.synchronize()
    finally:
        B.set_timeout_ns(old)
    assert int(status.item()) in TIMEOUT_CODES, f"no timeout reported (status {int(status.item())})"

    status.zero_()
    y = B.svdq_w4a4_gemm("nvfp4", codes, scales, lora, w, alpha, bias=bias, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref_pw = O.pack_weights("nvfp4", inp.W, inp.lam, inp.L1, inp.L2)
    act = O.quantize_activations("nvfp4", inp.x, ref_pw["inv_lam"], np.float32(inp.act_scale))
    y64 = O.linear_f64("nvfp4", act, ref_pw, inp.L1, inp.L2, inp.bias)
    assert_output_close(y.float().cpu().numpy(), y64, f"{kernel} GEMM after a timed-out call")


def test_int4_gemm_wait_timeout_reports_and_recovers():
    import bit_w4a4_diffusion_b200 as B
    # M = 4096: enough tiles per CTA that some wait outlasts the device
    # clock's resolution (the kernel is fast enough that at M = 1024 every
    # wait can end before the clock ticks).
    c = wl.SVDQ_CASES["int4_m4096"]
    inp = svdq_inputs(c)
    pk = B.svdq_pack_weights("int4", inp.W_bits, inp.lam, inp.L1_bits, inp.L2_bits)
    w = B.to_device(pk)
    x = B.bits_to_bf16(inp.x_bits, "cuda")
    codes, scales, lora = B.svdq_quantize_act("int4", x, w["inv_smooth"], w["lora_down"], 1.0, 1.0)
    torch.cuda.synchronize()

    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    old = B.get_timeout_ns()
    try:
        B.set_timeout_ns(1)
        B.svdq_w4a4_gemm("int4", codes, scales, lora, w, 1.0, dev_status=status)
        torch.cuda.synchronize()
    finally:
        B.set_timeout_ns(old)
    assert int(status.item()) in TIMEOUT_CODES, f"no timeout reported (status {int(status.item())})"

    status.zero_()
    y = B.svdq_w4a4_gemm("int4", codes, scales, lora, w, 1.0, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref_pw = O.pack_weights("int4", inp.W, inp.lam, inp.L1, inp.L2)
    act = O.quantize_activations("int4", inp.x, ref_pw["inv_lam"], np.float32(1.0))
    y64 = O.linear_f64("int4", act, ref_pw, inp.L1, inp.L2, inp.bias)
    assert_output_close(y.float().cpu().numpy(), y64, "INT4 GEMM after a timed-out call")


@pytest.mark.parametrize("option", ["default", "dq"])
def test_int4_layer_wait_timeout_reports_and_recovers(option, monkeypatch):
    """The INT4 layer's own GEMMs (the pair kernel on fp16 operands, and the
    one that builds the fp16 tiles itself) report a timed-out wait and leave
    the library usable."""
    import bit_w4a4_diffusion_b200 as B
    if option != "default":
        monkeypatch.setenv("SVDQ_INT4_LAYER_GEMM", option)
    c = wl.SVDQ_CASES["int4_m4096"]
    inp = svdq_inputs(c)
    pk = B.svdq_pack_weights("int4", inp.W_bits, inp.lam, inp.L1_bits, inp.L2_bits)
    w = B.to_device(pk)
    x = B.bits_to_bf16(inp.x_bits, "cuda")
    ws = torch.zeros(B.workspace_bytes("int4", c.M, c.N, c.K), dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    old = B.get_timeout_ns()
    try:
        B.set_timeout_ns(1)
        B.svdq_w4a4_linear("int4", x, w, 1.0, workspace=ws, dev_status=status)
        torch.cuda.synchronize()
    finally:
        B.set_timeout_ns(old)
    assert int(status.item()) in TIMEOUT_CODES, f"no timeout reported (status {int(status.item())})"

    status.zero_()
    y = B.svdq_w4a4_linear("int4", x, w, 1.0, workspace=ws, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref_pw = O.pack_weights("int4", inp.W, inp.lam, inp.L1, inp.L2)
    act = O.quantize_activations("int4", inp.x, ref_pw["inv_lam"])
    y64 = O.linear_f64("int4", act, ref_pw, inp.L1, inp.L2, inp.bias)
    assert_output_close(y.float().cpu().numpy(), y64, f"INT4 layer ({option}) after a timed-out call")


@pytest.mark.parametrize("kernel", ["single", "pair"])
def test_gelu_mlp_gemm_wait_timeout_reports_and_recovers(kernel, monkeypatch):
    """The GELU-MLP kernel (eight epilogue warps that stop together)."""
    monkeypatch.setenv("SVDQ_NVFP4_GEMM_KERNEL", kernel)
    import dataclasses
    import bit_w4a4_diffusion_b200 as B
    # K = 3072: thirteen K slices per tile, so that the load ring fills and
    # the waits last longer than the device clock's resolution.
    up = dataclasses.replace(wl.scaled_case(wl.SVDQ_CASES["mlp_up"], M=640, K=3072, N=1024), bias_std=0.1)
    dn = dataclasses.replace(wl.scaled_case(wl.SVDQ_CASES["mlp_down"], M=640, K=1024, N=768), bias_std=0.05)
    iu, idn = svdq_inputs(up), svdq_inputs(dn)
    pk_u = B.svdq_pack_weights("nvfp4", iu.W_bits, iu.lam, iu.L1_bits, iu.L2_bits)
    pk_d = B.svdq_pack_weights("nvfp4", idn.W_bits, idn.lam, idn.L1_bits, idn.L2_bits)
    wu, wd = B.to_device(pk_u), B.to_device(pk_d)
    x = B.bits_to_bf16(iu.x_bits, "cuda")
    b_u = B.bits_to_bf16(iu.bias_bits, "cuda")
    s_a = float(iu.act_scale)
    codes, scales, lora = B.svdq_quantize_act("nvfp4", x, wu["inv_smooth"], wu["lora_down"], s_a, wu["weight_scale_f"])
    alpha = float(np.float32(np.float32(s_a) * np.float32(pk_u["weight_scale"][0])))
    torch.cuda.synchronize()

    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    old = B.get_timeout_ns()
    try:
        B.set_timeout_ns(1)
        B.svdq_w4a4_gemm_gelu_quant(codes, scales, lora, wu, alpha, wd, float(idn.act_scale), bias=b_u,
                                    dev_status=status)
        torch.cuda.synchronize()
    finally:
        B.set_timeout_ns(old)
    assert int(status.item()) in TIMEOUT_CODES, f"no timeout reported (status {int(status.item())})"

    status.zero_()
    hc, hs, hl = B.svdq_w4a4_gemm_gelu_quant(codes, scales, lora, wu, alpha, wd, float(idn.act_scale), bias=b_u,
                                             dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    from tests.test_gpu_mlp import _check_hidden
    _check_hidden(iu, idn, pk_u, pk_d, hc, hs, hl)


@pytest.mark.parametrize("kernel", ["pair", "single"])
def test_qkv_gemm_wait_timeout_reports_and_recovers(kernel, monkeypatch):
    """The QKV + RMSNorm + RoPE kernel (eight epilogue warps that stop together)."""
    monkeypatch.setenv("SVDQ_NVFP4_GEMM_KERNEL", kernel)
    import bit_w4a4_diffusion_b200 as B
    from oracle import qkv as OQ
    M, K, heads = 640, 3072, 2       # thirteen K slices per tile, as above
    inp = svdq_inputs(wl.scaled_case(wl.SVDQ_CASES["qkv"], M=M, K=K, N=3 * heads * 128))
    pk = B.svdq_pack_weights("nvfp4", inp.W_bits, inp.lam, inp.L1_bits, inp.L2_bits)
    w = B.to_device(pk)
    gq, gk, cos, sin = wl.make_rope_norm_inputs(M, heads)
    d = [torch.from_numpy(np.ascontiguousarray(a)).cuda() for a in (gq, gk, cos.T, sin.T)]
    x = B.bits_to_bf16(inp.x_bits, "cuda")
    bias = B.bits_to_bf16(inp.bias_bits, "cuda")
    s_a = float(inp.act_scale)
    codes, scales, lora = B.svdq_quantize_act("nvfp4", x, w["inv_smooth"], w["lora_down"], s_a, w["weight_scale_f"])
    alpha = float(np.float32(np.float32(s_a) * np.float32(pk["weight_scale"][0])))
    torch.cuda.synchronize()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    old = B.get_timeout_ns()
    try:
        B.set_timeout_ns(1)
        B.svdq_w4a4_gemm_qkv_norm_rope(codes, scales, lora, w, alpha, heads, *d, bias=bias, dev_status=status)
        torch.cuda.synchronize()
    finally:
        B.set_timeout_ns(old)
    assert int(status.item()) in TIMEOUT_CODES, f"no timeout reported (status {int(status.item())})"
    status.zero_()
    y = B.svdq_w4a4_gemm_qkv_norm_rope(codes, scales, lora, w, alpha, heads, *d, bias=bias, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref_pw = O.pack_weights("nvfp4", inp.W, inp.lam, inp.L1, inp.L2)
    act = O.quantize_activations("nvfp4", inp.x, ref_pw["inv_lam"], np.float32(inp.act_scale))
    ref = OQ.qkv_layer_f64(act, ref_pw, inp.L1, inp.L2, inp.bias, gq, gk, cos, sin, heads)
    assert_output_close(y.float().cpu().numpy(), ref, "QKV GEMM after a timed-out call")


def test_timeout_through_the_default_binding_path_raises():
    """A call that passes no dev_status (the binding's default) reports to
    the library's own status word: a 1 ns wait limit makes the GEMM give up,
    and the next status check raises SvdqError(5); the check clears the
    word, and a normal call afterwards leaves it at 0."""
    import bit_w4a4_diffusion_b200 as B
    c = wl.scaled_case(wl.SVDQ_CASES["qkv"], M=640, N=2048)
    inp = svdq_inputs(c)
    pk = B.svdq_pack_weights("nvfp4", inp.W_bits, inp.lam, inp.L1_bits, inp.L2_bits)
    w = B.to_device(pk)
    x = B.bits_to_bf16(inp.x_bits, "cuda")
    s_a = float(inp.act_scale)
    torch.cuda.synchronize()
    assert B.device_status(clear=True) == 0
    old = B.get_timeout_ns()
    try:
        B.set_timeout_ns(1)
        B.svdq_w4a4_linear("nvfp4", x, w, s_a)
        torch.cuda.synchronize()
    finally:
        B.set_timeout_ns(old)
    with pytest.raises(B.SvdqError) as e:
        B.check_device_status()
    assert e.value.status == 5
    assert B.device_status(clear=False) == 0
    y = B.svdq_w4a4_linear("nvfp4", x, w, s_a)
    torch.cuda.synchronize()
    B.check_device_status()
    ref_pw = O.pack_weights("nvfp4", inp.W, inp.lam, inp.L1, inp.L2)
    act = O.quantize_activations("nvfp4", inp.x, ref_pw["inv_lam"], np.float32(inp.act_scale))
    y64 = O.linear_f64("nvfp4", act, ref_pw, inp.L1, inp.L2, None)
    assert_output_close(y.float().cpu().numpy(), y64, "layer after a timed-out call")


def test_fused_layer_wait_timeout_reports_and_recovers(monkeypatch):
    """The one-kernel layer (SVDQ_LAYER_KERNEL=fused): its producers wait
    (bounded) for row blocks that its epilogue warps quantize.  With a 1 ns
    limit some wait gives up; the kernel reports it, drains its copies, and
    its last CTA still returns the workspace's control words to zero, so the
    next call on the same workspace is correct."""
    import bit_w4a4_diffusion_b200 as B
    monkeypatch.setenv("SVDQ_LAYER_KERNEL", "fused")
    c = wl.scaled_case(wl.SVDQ_CASES["qkv"], M=640, N=2048)
    inp = svdq_inputs(c)
    pk = B.svdq_pack_weights("nvfp4", inp.W_bits, inp.lam, inp.L1_bits, inp.L2_bits)
    w = B.to_device(pk)
    bias = B.bits_to_bf16(inp.bias_bits, "cuda") if inp.bias_bits is not None else None
    x = B.bits_to_bf16(inp.x_bits, "cuda")
    s_a = float(inp.act_scale)
    ws = torch.zeros(B.workspace_bytes("nvfp4", c.M, c.N, c.K), dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    old = B.get_timeout_ns()
    try:
        B.set_timeout_ns(1)
        B.svdq_w4a4_linear("nvfp4", x, w, s_a, bias=bias, workspace=ws, dev_status=status)
        torch.cuda.synchronize()
    finally:
        B.set_timeout_ns(old)
    assert int(status.item()) in TIMEOUT_CODES, f"no timeout reported (status {int(status.item())})"
    off = B.workspace_offsets("nvfp4", c.M, c.N, c.K)
    assert int(ws[:off[1]].count_nonzero().item()) == 0, "control words not left at zero"
    status.zero_()
    y = B.svdq_w4a4_linear("nvfp4", x, w, s_a, bias=bias, workspace=ws, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref_pw = O.pack_weights("nvfp4", inp.W, inp.lam, inp.L1, inp.L2)
    act = O.quantize_activations("nvfp4", inp.x, ref_pw["inv_lam"], np.float32(inp.act_scale))
    y64 = O.linear_f64("nvfp4", act, ref_pw, inp.L1, inp.L2, inp.bias)
    assert_output_close(y.float().cpu().numpy(), y64, "one-kernel layer after a timed-out call")
