"""GPU parity: the CUDA SVDQuant W4A4 path against the CPU oracle.

Activation codes and group scales must match the oracle bit for bit; the
layer output must satisfy the bound in ``helpers.assert_output_close``.
Small cases (every output checked) span several tiles with ragged M / N
tails; the full-size workloads compare every activation code and a sample of
output rows the oracle computes one by one.
"""
import numpy as np
import pytest
import torch

import workloads as wl
from oracle import svdq as O
from tests.helpers import assert_output_close, nibbles, svdq_inputs

pytestmark = pytest.mark.gpu

B = None


def _lib():
    global B
    if B is None:
        import bit_w4a4_diffusion_b200 as _B
        B = _B
    return B


def _run_s1(inp, w, prec="nvfp4"):
    B = _lib()
    x = B.bits_to_bf16(inp.x_bits, "cuda")
    s_a = float(inp.act_scale)
    codes, scales, lora = B.svdq_quantize_act(prec, x, w["inv_smooth"], w["lora_down"], s_a, w["weight_scale_f"])
    return x, codes, scales, lora


def _check_s1(inp, codes, scales, lora, pk, rows=None):
    """Bit-exact codes / scales (all rows or `rows`), and the low-rank activation."""
    c = inp.case
    M, K = c.M, c.K
    inv = O.inverse_smoothing(inp.lam)
    sel = slice(None) if rows is None else rows
    xs = inp.x if rows is None else inp.x[rows]
    ref = O.quantize_activations("nvfp4", xs, inv, np.float32(inp.act_scale))
    got_codes = nibbles(codes.cpu().numpy())[sel]
    assert np.array_equal(got_codes, ref["codes"]), "activation codes differ"
    sc_all = _lib().scales_to_rowmajor(scales.cpu().numpy(), M, K)
    assert np.array_equal(sc_all[sel], ref["scales"]), "activation scales differ"
    # padding rows of the tiled scale layout are zero
    Mp = (M + 255) // 256 * 256
    if Mp > M:
        full = _lib().scales_to_rowmajor(scales.cpu().numpy(), Mp, K)
        assert np.all(full[M:] == 0)
    # low-rank activation: hi + lo = u / alpha with u = x_hat L1 (fp16 operands:
    # 11-bit significands, fp32 accumulation)
    alpha = np.float64(np.float32(np.float32(inp.act_scale) * np.float32(pk["weight_scale"][0])))
    la = lora.float().cpu().numpy().astype(np.float64)[sel]
    u = ref["x_hat"].astype(np.float64) @ inp.L1.astype(np.float64) / alpha
    err = np.abs(la[:, :32] + la[:, 32:] - u)
    assert np.max(err) <= 2e-3 * np.max(np.abs(u)) + 1e-30, f"low-rank activation error {np.max(err)}"
    assert np.linalg.norm(err) <= 5e-4 * np.linalg.norm(u) + 1e-30
    return ref


def _layer(c):
    B = _lib()
    inp = svdq_inputs(c)
    pk = B.svdq_pack_weights("nvfp4", inp.W_bits, inp.lam, inp.L1_bits, inp.L2_bits)
    w = B.to_device(pk)
    bias = B.bits_to_bf16(inp.bias_bits, "cuda") if inp.bias_bits is not None else None
    return inp, pk, w, bias


def _check_layer_workspace(ws, c, codes, scales, lora):
    """The layer's workspace after a call: activation codes and scales equal
    the quantize kernel's bit for bit, the low-rank activation equal up to the
    order of its fp32 sums, and the control words back at zero."""
    B = _lib()
    off = B.workspace_offsets("nvfp4", c.M, c.N, c.K)
    wcodes = ws[off[1]:off[1] + c.M * c.K // 2].view(c.M, c.K // 2)
    wscales = ws[off[2]:off[2] + B.act_scale_bytes("nvfp4", c.M, c.K)]
    wlora = ws[off[3]:off[3] + c.M * 128].view(torch.bfloat16).view(c.M, 64)
    assert torch.equal(wcodes, codes), "layer codes differ from the quantize kernel's"
    assert torch.equal(wscales, scales), "layer scales differ from the quantize kernel's"
    ua = wlora.double()[:, :32] + wlora.double()[:, 32:]
    ub = lora.double()[:, :32] + lora.double()[:, 32:]
    # fp32 sums of the same products in two orders (the oracle bound on u is 2e-3 max|u|)
    assert (ua - ub).abs().max().item() <= 1e-4 * ub.abs().max().item() + 1e-30
    assert int(ws[:off[1]].count_nonzero().item()) == 0, "control words not left at zero"


SMALL = [
    ("tiny", {}),
    ("qkv", dict(M=300, N=1024)),          # ragged M, bias, weight outliers
    ("mlp_up", dict(M=384, N=384)),        # N % 256 == 128 (half tile)
    ("mlp_down", dict(M=200, N=512)),      # K = 12288, GELU activations
    ("tiny", dict(M=1, N=256)),            # a single token
    ("qkv", dict(M=129, N=2048, K=1024)),  # one row past a tile
]


@pytest.mark.parametrize("kernel", ["pair", "single", "fused"])
@pytest.mark.parametrize("name,kw", SMALL)
def test_linear_small_matches_oracle(name, kw, kernel, monkeypatch):
    """Both NVFP4 GEMM kernels: the CTA-pair kernel (the default) and the
    one-CTA-per-tile kernel, with the layer as quantize + GEMM; and the
    one-kernel layer (SVDQ_LAYER_KERNEL=fused), which quantizes x inside the
    pair GEMM."""
    monkeypatch.setenv("SVDQ_NVFP4_GEMM_KERNEL", "single" if kernel == "single" else "pair")
    if kernel == "fused":
        monkeypatch.setenv("SVDQ_LAYER_KERNEL", "fused")
    B = _lib()
    c = wl.SVDQ_CASES[name]
    if kw:
        c = wl.scaled_case(c, **kw)
    inp, pk, w, bias = _layer(c)
    x, codes, scales, lora = _run_s1(inp, w)
    alpha = float(np.float32(np.float32(inp.act_scale) * np.float32(pk["weight_scale"][0])))
    y = B.svdq_w4a4_gemm("nvfp4", codes, scales, lora, w, alpha, bias=bias)
    ws = torch.zeros(B.workspace_bytes("nvfp4", c.M, c.N, c.K), dtype=torch.uint8, device="cuda")
    y2 = B.svdq_w4a4_linear("nvfp4", x, w, float(inp.act_scale), bias=bias, workspace=ws)
    torch.cuda.synchronize()
    _check_s1(inp, codes, scales, lora, pk)
    ref_pw = O.pack_weights("nvfp4", inp.W, inp.lam, inp.L1, inp.L2)
    act = O.quantize_activations("nvfp4", inp.x, ref_pw["inv_lam"], np.float32(inp.act_scale))
    y64 = O.linear_f64("nvfp4", act, ref_pw, inp.L1, inp.L2, inp.bias)
    yg = y.float().cpu().numpy()
    assert_output_close(yg, y64, f"{c.name} gemm")
    _check_layer_workspace(ws, c, codes, scales, lora)
    if kernel != "fused":
        # the two-kernel path: the layer is quantize + gemm, bit for bit
        assert torch.equal(y, y2), "svdq_w4a4_linear differs from quantize + gemm"
    else:
        # one kernel: the low-rank sums run in another (fixed) order
        assert_output_close(y2.float().cpu().numpy(), y64, f"{c.name} layer")


@pytest.mark.parametrize("name,kw", SMALL)
def test_quantizers_agree(name, kw, monkeypatch):
    """The TMA-fed NVFP4 quantizer (the default) and the per-thread-copy one
    produce the same codes and scales bit for bit; their low-rank activations
    differ only by the order of the fp32 partial sums (each is checked
    against the oracle in the other tests)."""
    B = _lib()
    c = wl.SVDQ_CASES[name]
    if kw:
        c = wl.scaled_case(c, **kw)
    inp, pk, w, bias = _layer(c)
    outs = {}
    for kern in ("tma", "copy"):
        monkeypatch.setenv("SVDQ_NVFP4_QUANT_KERNEL", kern)
        outs[kern] = _run_s1(inp, w)[1:]
    torch.cuda.synchronize()
    for a, b, what in zip(outs["tma"][:2], outs["copy"][:2], ("codes", "scales")):
        assert torch.equal(a, b), f"{c.name}: {what} differ between the two quantizers"
    la = outs["tma"][2].float().cpu().numpy()
    lb = outs["copy"][2].float().cpu().numpy()
    u_a, u_b = la[:, :32] + la[:, 32:], lb[:, :32] + lb[:, 32:]
    assert np.max(np.abs(u_a - u_b)) <= 1e-5 * np.max(np.abs(u_b)) + 1e-30


def test_quantize_ties_and_signed_zero():
    """Exact E2M1 midpoints and values that round to -0 (inv_smooth = 1)."""
    B = _lib()
    K = 256
    s_a = np.float32(2.0 ** -8)
    ratios = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0,
                       -0.25, -0.75, -1.25, -1.75, -2.5, -3.5, -5.0, -2.0 ** -10], np.float32)
    x = np.zeros((16, K), np.float32)
    for r in range(16):
        x[r] = np.roll(np.tile(ratios, K // 16), r) * s_a      # each group holds +-6 or 6 -> scale 1.0
    x[3, 32:48] = 0.0                                          # a zero group
    bits, xv = wl.to_bf16(x)
    assert np.array_equal(xv, x)
    dev = "cuda"
    xd = B.bits_to_bf16(bits, dev)
    inv = torch.ones(K, dtype=torch.float32, device=dev)
    l1t = torch.zeros((32, K), dtype=torch.bfloat16, device=dev)
    codes, scales, lora = B.svdq_quantize_act("nvfp4", xd, inv, l1t, float(s_a), 1.0)
    torch.cuda.synchronize()
    ref = O.quantize_activations("nvfp4", xv, np.ones(K, np.float32), s_a)
    assert np.array_equal(nibbles(codes.cpu().numpy()), ref["codes"])
    assert np.array_equal(B.scales_to_rowmajor(scales.cpu().numpy(), 16, K), ref["scales"])
    assert np.all(lora.float().cpu().numpy() == 0)


def _order_case_inputs(vals, K_mult=256):
    """One long row of case values as 1/lambda (x = +-1, 0.5 then gives
    x_hat = +-vals, vals / 2 exactly)."""
    K = -(-vals.size // K_mult) * K_mult
    inv = np.zeros(K, np.float32)
    inv[:vals.size] = vals
    x = np.zeros((3, K), np.float32)
    x[0], x[1], x[2] = 1.0, -1.0, 0.5
    bits, xv = wl.to_bf16(x)
    assert np.array_equal(xv, x)
    return K, inv, bits, xv


@pytest.mark.parametrize("s_a", [0.0123457, 3.1e-5])
def test_quantize_operation_order_cases(s_a):
    """Inputs on which fl(v * fl(1/d)) and fl(v / d) give different E2M1
    codes, or fl(a * fl(1/(6 s))) and fl(a / (6 s)) different E4M3 scale
    bytes, under a tensor scale whose reciprocals are inexact: the device
    codes and scales equal the oracle's (the reciprocal form) bit for bit."""
    from tests import quant_order_cases as QC
    B = _lib()
    s = np.float32(s_a)
    rows, where = QC.nvfp4_rows(s)
    assert len(where) >= 48
    K, inv, bits, xv = _order_case_inputs(rows.reshape(-1))
    dev = "cuda"
    codes, scales, lora = B.svdq_quantize_act("nvfp4", B.bits_to_bf16(bits, dev), torch.from_numpy(inv).to(dev),
                                              torch.zeros((32, K), dtype=torch.float16, device=dev), float(s), 1.0)
    torch.cuda.synchronize()
    ref = O.quantize_activations("nvfp4", xv, inv, s)
    assert np.array_equal(nibbles(codes.cpu().numpy()), ref["codes"])
    assert np.array_equal(B.scales_to_rowmajor(scales.cpu().numpy(), 3, K), ref["scales"])
    assert np.all(lora.float().cpu().numpy() == 0)


def test_quantize_int4_operation_order_cases():
    """INT4: inputs on which rint(fl(v * fl(1/sc))) and rint(fl(v / sc))
    differ; the device codes and bf16 scales equal the oracle's."""
    from tests import quant_order_cases as QC
    B = _lib()
    rows, where = QC.int4_rows(32)
    assert len(where) >= 24
    K, inv, bits, xv = _order_case_inputs(rows.reshape(-1))
    dev = "cuda"
    codes, scales, lora = B.svdq_quantize_act("int4", B.bits_to_bf16(bits, dev), torch.from_numpy(inv).to(dev),
                                              torch.zeros((32, K), dtype=torch.bfloat16, device=dev), 1.0, 1.0)
    torch.cuda.synchronize()
    ref = O.quantize_activations("int4", xv, inv)
    got = nibbles(codes.cpu().numpy()).astype(np.int16)
    got = np.where(got >= 8, got - 16, got)
    assert np.array_equal(got, ref["q"].astype(np.int16))
    sc = scales.cpu().numpy().view(np.uint16).reshape(K // 64, -1)[:, :3].T
    assert np.array_equal(wl.to_bf16(ref["sc"])[0], sc)


FULL = ["qkv", "mlp_up", "mlp_down"]


@pytest.mark.parametrize("kernel", ["single", "pair", "fused"])
@pytest.mark.parametrize("name", FULL)
def test_linear_full_size_sampled(name, kernel, monkeypatch):
    """Full workload shape (the launch configuration the benchmark times):
    all activation codes bit-exact, 48 sampled output rows within tolerance."""
    monkeypatch.setenv("SVDQ_NVFP4_GEMM_KERNEL", "single" if kernel == "single" else "pair")
    if kernel == "fused":
        monkeypatch.setenv("SVDQ_LAYER_KERNEL", "fused")
    B = _lib()
    c = wl.SVDQ_CASES[name]
    inp, pk, w, bias = _layer(c)
    x = B.bits_to_bf16(inp.x_bits, "cuda")
    ws = torch.zeros(B.workspace_bytes("nvfp4", c.M, c.N, c.K), dtype=torch.uint8, device="cuda")
    y = B.svdq_w4a4_linear("nvfp4", x, w, float(inp.act_scale), bias=bias, workspace=ws)
    y_again = B.svdq_w4a4_linear("nvfp4", x, w, float(inp.act_scale), bias=bias, workspace=ws)
    _, codes, scales, lora = _run_s1(inp, w)
    torch.cuda.synchronize()
    ref = _check_s1(inp, codes, scales, lora, pk)
    _check_layer_workspace(ws, c, codes, scales, lora)
    assert torch.equal(y, y_again), "the layer is not deterministic"
    rng = np.random.default_rng(99)
    rows = np.sort(np.concatenate([[0, c.M - 1], rng.choice(np.arange(1, c.M - 1), 46, replace=False)]))
    act = {k: ref[k][rows] for k in ("codes", "scales", "x_hat")}
    act["s_a"] = np.float32(inp.act_scale)
    ref_pw = O.pack_weights("nvfp4", inp.W, inp.lam, inp.L1, inp.L2)
    y64 = O.linear_f64("nvfp4", act, ref_pw, inp.L1, inp.L2, inp.bias)
    yg = y.float().cpu().numpy()[rows]
    assert_output_close(yg, y64, f"{name} full (sampled rows)")


def test_gemm_rejects_unsupported_shapes_before_launch():
    B = _lib()
    x = torch.zeros((4, 100), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(B.SvdqError) as e:
        B.svdq_quantize_act("nvfp4", x, torch.ones(100, device="cuda"),
                            torch.zeros((32, 100), dtype=torch.bfloat16, device="cuda"), 1.0, 1.0)
    assert e.value.status == 2
