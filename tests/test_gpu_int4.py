"""GPU parity: the CUDA SVDQuant W4A4 INT4 path (S1 INT4 quantize + S3 i8
tcgen05 GEMM) against the CPU oracle.  Activation codes and bf16 group scales
bit-exact; outputs within the layer bound; every output row checked."""
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
    y2 = B.svdq_w4a4_linear("int4", x, w, 1.0)
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
    assert torch.equal(y, y2)
