"""GPU parity: the CUDA SVDQuant W4A4 INT4 path against the CPU oracle.  S1
(INT4 quantize): activation codes and bf16 group scales bit-exact.  S3 three
ways: svdq_w4a4_gemm's i8 tcgen05 kernel; the layer's default, the fp16
tensor pipe on fp16 operands written out first, whose values must be exactly
the oracle's dequantized codes (scaled by the documented power of two per
row); and the same product with the fp16 operand tiles built inside the
GEMM.  The two fp16 paths issue the same MMAs on the same values and must
agree bit for bit.  Outputs within the layer bound; every output row
checked."""
import numpy as np
import pytest
import torch

import workloads as wl
from oracle import svdq as O
from tests.helpers import assert_output_close, nibbles, svdq_inputs

pytestmark = pytest.mark.gpu


def _int4_codes(packed):
    q = nibbles(packed).astype(np.int8)
    return np.where(q > 7, q - 16, q).astype(np.int8)


CASES = [
    ("int4_m1024", dict(M=300, N=512)),                 # ragged M
    ("int4_m1024", dict(M=129, N=256, K=1024)),
    ("int4_m1024", dict(M=1, N=128, K=256)),             # one token, one tile
    ("int4_m1024", dict(M=130, N=384, K=512)),           # half of the last 256-column tile past N
    ("int4_m1024", {}),
    ("int4_m2048", {}),
    ("int4_m4096", {}),
    ("int4_m8192", {}),
]


@pytest.mark.parametrize("name,kw", CASES)
def test_int4_linear_matches_oracle(name, kw):
    import bit_w4a4_diffusion_b200 as B
    c = wl.SVDQ_CASES[name]
    if kw:
        c = wl.scaled_case(c, **kw)
    inp = svdq_inputs(c)
    pk = B.svdq_pack_weights("int4", inp.W_bits, inp.lam, inp.L1_bits, inp.L2_bits)
    w = B.to_device(pk)
    x = B.bits_to_bf16(inp.x_bits, "cuda")
    codes, scales, lora = B.svdq_quantize_act("int4", x, w["inv_smooth"], w["lora_down"], 1.0, 1.0)
    y = B.svdq_w4a4_gemm("int4", codes, scales, lora, w, 1.0)
    y2 = B.svdq_w4a4_linear("int4", x, w, 1.0)              # fp16 operands written out first
    with _env("SVDQ_INT4_LAYER_GEMM", "i8"):
        y3 = B.svdq_w4a4_linear("int4", x, w, 1.0)          # the i8 kernel
    with _env("SVDQ_INT4_LAYER_GEMM", "dq"):
        y4 = B.svdq_w4a4_linear("int4", x, w, 1.0)          # fp16 tiles built in the GEMM
    torch.cuda.synchronize()
    ref_pw = O.pack_weights("int4", inp.W, inp.lam, inp.L1, inp.L2)
    act = O.quantize_activations("int4", inp.x, ref_pw["inv_lam"])
    assert np.array_equal(_int4_codes(codes.cpu().numpy()), act["q"]), "activation codes differ"
    Mp = (c.M + 255) // 256 * 256
    sc = scales.cpu().numpy().view(np.uint16).reshape(c.K // 64, Mp)
    assert np.array_equal(sc[:, :c.M].T, wl.to_bf16(act["sc"])[0]), "activation scales differ"
    assert np.all(sc[:, c.M:] == 0)
    la = lora.float().cpu().numpy().astype(np.float64)
    u = act["x_hat"].astype(np.float64) @ inp.L1.astype(np.float64)
    assert np.max(np.abs(la[:, :32] + la[:, 32:] - u)) <= 1e-5 * np.max(np.abs(u))
    y64 = O.linear_f64("int4", act, ref_pw, inp.L1, inp.L2, inp.bias)
    assert_output_close(y.float().cpu().numpy(), y64, f"{c.name} int4")
    assert_output_close(y2.float().cpu().numpy(), y64, f"{c.name} int4 (fp16 operands)")
    assert torch.equal(y, y3)
    assert torch.equal(y2, y4), "the two fp16 paths differ"
    # Both products sum the same exact terms in fp32, in different orders:
    # they differ by fp32 rounding (a few 2^-24 of the terms' magnitudes, far
    # below 2^-12 of the output's largest) and then by at most one bf16 step.
    d = (y.float() - y2.float()).abs()
    bound = torch.maximum(y.float().abs(), y2.float().abs()) * 2.0 ** -7 + float(y.float().abs().max()) * 2.0 ** -12
    assert bool((d <= bound).all()), f"fp16-operand and i8 products differ by up to {float((d / bound).max()):.2f}x the bound"


class _env:
    """Set an environment variable for the duration of a with block."""

    def __init__(self, key, value):
        self.key, self.value = key, value

    def __enter__(self):
        import os
        self.old = os.environ.get(self.key)
        os.environ[self.key] = self.value

    def __exit__(self, *exc):
        import os
        if self.old is None:
            os.environ.pop(self.key, None)
        else:
            os.environ[self.key] = self.old


# Position p of every 8-element block of an fp16 operand row holds element
# PERM[p] of the block.
PERM = np.array([0, 2, 4, 6, 1, 3, 5, 7])


def _expected_fp16(q, sc):
    """The fp16 operand rows the layer must build from INT4 codes q [R, K]
    and group scales sc [R, K/64] (fp32 holding bf16 values): row r scaled by
    2^-E[r], E[r] = floor(log2(max_g sc[r, g])) - 12 clamped to [-100, 100]
    (0 for a zero row), every value exact in fp16 when its group's scale is
    within 2^29 of the row's largest.  Returns (fp16 [R, K], 2^E [R])."""
    sc = np.asarray(sc, np.float64)
    mx = sc.max(axis=1)
    _, e2 = np.frexp(np.where(mx > 0, mx, 1.0))        # mx = f 2^e2, f in [0.5, 1)
    E = np.where(mx > 0, np.clip(e2 - 1 - 12, -100, 100), 0)
    v = np.repeat(sc, 64, axis=1) * np.ldexp(1.0, -E)[:, None] * np.asarray(q, np.float64)
    return v.astype(np.float16), np.ldexp(1.0, E).astype(np.float32)


def _unpermute(a16):
    R, K = a16.shape
    out = np.empty_like(a16)
    out.reshape(R, K // 8, 8)[:, :, PERM] = a16.reshape(R, K // 8, 8)
    return out


@pytest.mark.parametrize("name,kw,zero_row", [("int4_m1024", dict(M=300, N=512), 7),
                                              ("int4_m1024", dict(M=129, N=256, K=1024), None),
                                              ("int4_m2048", {}, 1000),   # weight rows in the quantizer's launch
                                              ("int4_m4096", {}, None)])  # both sides in the operand pass
def test_int4_fp16_operands_are_the_oracle_values(name, kw, zero_row):
    """The layer's fp16 operands (workspace region [4]) against the oracle's
    codes and scales, bit for bit: A' from the activation quantizer, W' from
    the weight pack, and the rows' powers of two (which the "dq" option
    computes the same way).  A row of
    x set to zero checks the zero-row case (factor 1, all values +0)."""
    import bit_w4a4_diffusion_b200 as B
    c = wl.SVDQ_CASES[name]
    if kw:
        c = wl.scaled_case(c, **kw)
    inp = svdq_inputs(c)
    x_bits = inp.x_bits.copy()
    x_f = inp.x.copy()
    if zero_row is not None:
        x_bits[zero_row] = 0
        x_f[zero_row] = 0.0
    pk = B.svdq_pack_weights("int4", inp.W_bits, inp.lam, inp.L1_bits, inp.L2_bits)
    w = B.to_device(pk)
    x = B.bits_to_bf16(x_bits, "cuda")
    ws = torch.zeros(B.workspace_bytes("int4", c.M, c.N, c.K), dtype=torch.uint8, device="cuda")
    y = B.svdq_w4a4_linear("int4", x, w, 1.0, workspace=ws)
    with _env("SVDQ_INT4_LAYER_GEMM", "dq"):
        y_dq = B.svdq_w4a4_linear("int4", x, w, 1.0)
    torch.cuda.synchronize()
    assert torch.equal(y, y_dq), "the two fp16 paths differ"
    off = B.workspace_offsets("int4", c.M, c.N, c.K)
    region = ws[off[4]:off[5]].cpu().numpy()

    def at(o, nbytes):
        return region[o:o + nbytes]

    M, N, K = c.M, c.N, c.K
    r256 = lambda v: -(-v // 256) * 256
    o_a, o_fa = 0, r256(M * K * 2) + r256(M * 128)
    o_w = o_fa + r256(M * 4)
    o_fw = o_w + r256(N * K * 2) + r256(N * 128)
    a16 = _unpermute(at(o_a, M * K * 2).view(np.float16).reshape(M, K))
    fa = at(o_fa, M * 4).view(np.float32)
    w16 = _unpermute(at(o_w, N * K * 2).view(np.float16).reshape(N, K))
    fw = at(o_fw, N * 4).view(np.float32)

    ref_pw = O.pack_weights("int4", inp.W, inp.lam, inp.L1, inp.L2)
    act = O.quantize_activations("int4", x_f, ref_pw["inv_lam"])
    ea, efa = _expected_fp16(act["q"], act["sc"])
    ew, efw = _expected_fp16(ref_pw["q"], ref_pw["sc"])
    assert np.array_equal(a16.view(np.uint16), ea.view(np.uint16)), "activation fp16 operand differs"
    assert np.array_equal(fa, efa), "activation row powers of two differ"
    assert np.array_equal(w16.view(np.uint16), ew.view(np.uint16)), "weight fp16 operand differs"
    assert np.array_equal(fw, efw), "weight row powers of two differ"
    if zero_row is not None:
        assert fa[zero_row] == 1.0 and not a16[zero_row].view(np.uint16).any()
    y64 = O.linear_f64("int4", act, ref_pw, inp.L1, inp.L2, inp.bias)
    assert_output_close(y.float().cpu().numpy(), y64, f"{c.name} int4 fp16 operands")
