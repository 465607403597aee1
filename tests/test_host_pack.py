"""The library's C++ host packer against the oracle (CPU only, bit-exact).

Two independent implementations of the offline weight preparation (the
oracle's numpy code and the library's C++) must agree bit for bit on the
residual's quantized codes, the group scales, the tensor scale and the
inverse smoothing vector.
"""
import numpy as np
import pytest

import bit_w4a4_diffusion_b200 as B
import workloads as wl
from tests.helpers import svdq_inputs
from oracle import awq as OA
from oracle import svdq as O


def _nibbles(packed):
    lo = packed & 0xF
    hi = packed >> 4
    return np.stack([lo, hi], axis=-1).reshape(packed.shape[0], -1)


CASES = [
    ("tiny", {}),
    ("qkv", dict(M=64, N=1024, K=3072)),
    ("mlp_down", dict(M=64, N=384, K=2048)),
    ("int4_m1024", dict(M=64, N=512, K=1024)),
]


@pytest.mark.parametrize("name,kw", CASES)
def test_pack_weights_matches_oracle(name, kw):
    c = wl.SVDQ_CASES[name]
    if kw:
        c = wl.scaled_case(c, **kw)
    inp = svdq_inputs(c)
    pk = B.svdq_pack_weights(c.precision, inp.W_bits, inp.lam, inp.L1_bits, inp.L2_bits)
    ref = O.pack_weights(c.precision, inp.W, inp.lam, inp.L1, inp.L2)
    assert np.array_equal(pk["inv_smooth"], ref["inv_lam"])
    if c.precision == "nvfp4":
        assert pk["weight_scale"][0] == ref["s_w"]
        assert np.array_equal(_nibbles(pk["codes"]), ref["codes"])
        assert np.array_equal(B.scales_to_rowmajor(pk["scales"], c.N, c.K), ref["scales"])
        # padding rows of the tiled layout are zero
        tiled_again = B.scales_from_rowmajor(ref["scales"], c.N, c.K)
        assert np.array_equal(tiled_again, pk["scales"])
    else:
        q = _nibbles(pk["codes"]).astype(np.int8)
        q = np.where(q > 7, q - 16, q).astype(np.int8)
        assert np.array_equal(q, ref["q"])
        np_ = (c.N + 255) // 256 * 256
        sc = pk["scales"].view(np.uint16).reshape(c.K // 64, np_)[:, :c.N].T
        assert np.array_equal(wl.to_bf16(ref["sc"])[0], sc)
    # low-rank operand layouts (the NVFP4 down-projection operand is fp16)
    if c.precision == "nvfp4":
        assert pk["lora_down"].dtype == np.float16
        assert np.array_equal(pk["lora_down"], inp.L1.T.astype(np.float16))
    else:
        assert np.array_equal(pk["lora_down"], inp.L1_bits.T)
    assert np.array_equal(pk["lora_up"][:, :32], inp.L2_bits.T)
    assert np.array_equal(pk["lora_up"][:, 32:], inp.L2_bits.T)


def test_pack_rejects_bad_shapes():
    W = np.zeros((100, 256), np.uint16)
    with pytest.raises(B.SvdqError):
        B.svdq_pack_weights("nvfp4", W, np.ones(256, np.float32), np.zeros((256, 32), np.uint16),
                            np.zeros((32, 100), np.uint16))


def test_scale_layout_formula_round_trip():
    rng = np.random.default_rng(5)
    rows, K = 300, 512
    rm = rng.integers(0, 127, (rows, K // 16)).astype(np.uint8)
    tiled = B.scales_from_rowmajor(rm, rows, K)
    assert tiled.size == 512 * (K // 16)
    # spot-check the documented offset formula
    for (m, g) in [(0, 0), (37, 5), (129, 31), (299, 17)]:
        off = ((m // 128) * (K // 64) + g // 4) * 512 + (m % 32) * 16 + ((m % 128) // 32) * 4 + g % 4
        assert tiled[off] == rm[m, g]
    assert np.array_equal(B.scales_to_rowmajor(tiled, rows, K), rm)


@pytest.mark.parametrize("N,K", [(64, 256), (18432 // 16, 3072)])
def test_awq_pack_matches_oracle(N, K):
    inp = wl.make_awq_inputs(2, N=N, K=K)
    pk = B.awq_pack_weights(inp.W_bits)
    q, sc, z = OA.awq_quantize(inp.W)
    assert np.array_equal(_nibbles(pk["qweight"]), q)
    assert np.array_equal(pk["scales"], wl.to_bf16(sc)[0])
    zz = np.stack([pk["zeros"] & 0xF, pk["zeros"] >> 4], axis=-1).reshape(N, -1)
    assert np.array_equal(zz, z)


def test_fp16_operand_rounding_matches_numpy():
    """The packer's bf16 -> fp16 conversion of L1 (every finite bf16 value up
    to 65504, subnormal range included) against numpy's float16 cast."""
    bits = np.arange(0, 0x8000, dtype=np.uint32).astype(np.uint16)
    vals = (bits.astype(np.uint32) << 16).view(np.float32)
    keep = np.isfinite(vals) & (vals <= 65504.0)
    vals = vals[keep]
    K = 256
    n = (len(vals) // K) * K
    L1 = np.concatenate([vals[:n], -vals[:n]]).reshape(-1, K)[:, :K]
    L1 = L1[: (L1.shape[0] // 32) * 32]
    r_blocks = L1.reshape(-1, 32, K)
    for blk in r_blocks[:: max(1, len(r_blocks) // 40)]:
        L1b = wl.to_bf16(blk.T.astype(np.float32))[0]           # [K, 32] bits
        pk = B.svdq_pack_weights("nvfp4", np.zeros((128, K), np.uint16), np.ones(K, np.float32), L1b,
                                 np.zeros((32, 128), np.uint16))
        assert np.array_equal(pk["lora_down"].view(np.uint16), blk.astype(np.float16).view(np.uint16))


def test_pack_rejects_out_of_fp16_range_factor():
    L1 = np.zeros((256, 32), np.float32)
    L1[3, 5] = 70000.0
    with pytest.raises(B.SvdqError):
        B.svdq_pack_weights("nvfp4", np.zeros((128, 256), np.uint16), np.ones(256, np.float32),
                            wl.to_bf16(L1)[0], np.zeros((32, 128), np.uint16))


# The five workloads at their full weight shapes: the per-tensor scale s_w
# depends on the whole residual, so a scaled-down shape does not stand in for
# the full one.
FULL = ["qkv", "mlp_up", "mlp_down", "int4_m1024"]


@pytest.mark.slow
@pytest.mark.parametrize("name", FULL)
def test_pack_weights_matches_oracle_full_size(name):
    c = wl.SVDQ_CASES[name]
    inp = svdq_inputs(c)
    pk = B.svdq_pack_weights(c.precision, inp.W_bits, inp.lam, inp.L1_bits, inp.L2_bits)
    ref = O.pack_weights(c.precision, inp.W, inp.lam, inp.L1, inp.L2)
    assert np.array_equal(pk["inv_smooth"], ref["inv_lam"])
    if c.precision == "nvfp4":
        assert pk["weight_scale"][0] == ref["s_w"]
        assert np.array_equal(_nibbles(pk["codes"]), ref["codes"])
        assert np.array_equal(B.scales_to_rowmajor(pk["scales"], c.N, c.K), ref["scales"])
    else:
        q = _nibbles(pk["codes"]).astype(np.int8)
        assert np.array_equal(np.where(q > 7, q - 16, q).astype(np.int8), ref["q"])
        np_ = (c.N + 255) // 256 * 256
        sc = pk["scales"].view(np.uint16).reshape(c.K // 64, np_)[:, :c.N].T
        assert np.array_equal(wl.to_bf16(ref["sc"])[0], sc)


@pytest.mark.slow
def test_awq_pack_matches_oracle_full_size():
    inp = wl.make_awq_inputs(1)                       # W [18432, 3072]
    pk = B.awq_pack_weights(inp.W_bits)
    q, sc, z = OA.awq_quantize(inp.W)
    assert np.array_equal(_nibbles(pk["qweight"]), q)
    assert np.array_equal(pk["scales"], wl.to_bf16(sc)[0])
    zz = np.stack([pk["zeros"] & 0xF, pk["zeros"] >> 4], axis=-1).reshape(inp.N, -1)
    assert np.array_equal(zz, z)
