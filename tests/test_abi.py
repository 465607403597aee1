"""The C ABI on the host: every symbol declared in include/svdq.h is exported
by the built library, and argument errors are reported before anything is
launched (no GPU needed; no call here reaches a kernel launch)."""
import ctypes
import os
import re

import pytest

import bit_w4a4_diffusion_b200 as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if not fn.endswith(".h"):
            continue
        text = open(os.path.join(ROOT, "include", fn)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^[A-Za-z_][\w \*]*?\b([a-z_][a-z0-9_]*)\s*\(", text, flags=re.M):
            names.append(m.group(1))
    return sorted(set(names))


def test_header_symbols_are_exported():
    names = _declared_functions()
    assert "svdq_w4a4_linear" in names and "awq_w4a16_linear" in names and "svdq_pack_weights" in names
    lib = ctypes.CDLL(B.LIB_PATH)
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, f"declared but not exported: {missing}"


def test_status_strings_and_version():
    assert B.lib.svdq_version() >= 1
    assert B.lib.svdq_status_string(0) == b"ok"
    assert B.lib.svdq_status_string(2) == b"unsupported shape"


def test_sizes():
    assert B.act_scale_bytes("nvfp4", 4096, 3072) == 4096 * 3072 // 16
    assert B.act_scale_bytes("nvfp4", 300, 1024) == 512 * 1024 // 16
    assert B.act_scale_bytes("int4", 300, 1024) == 512 * 1024 // 64 * 2
    assert B.act_scale_bytes(7, 300, 1024) == -1
    assert B.workspace_bytes("nvfp4", 4096, 12288, 3072) >= 4096 * 1536 + 4096 * 192 + 4096 * 128
    assert B.workspace_bytes("nvfp4", 4096, 12288, 3072, rank=16) == -1
    # NVFP4 workspaces do not depend on N; INT4 ones hold the fp16 operands
    # A' [M, K] and W' [N, K] besides the quantized activations.
    assert B.workspace_bytes("nvfp4", 4096, 0, 3072) == B.workspace_bytes("nvfp4", 4096, 12288, 3072)
    base = B.workspace_offsets("int4", 4096, 3072, 3072)
    assert base[5] - base[4] >= (4096 + 3072) * 3072 * 2 + (4096 + 3072) * (128 + 4)
    assert B.workspace_bytes("int4", 4096, 6144, 3072) - B.workspace_bytes("int4", 4096, 3072, 3072) == 3072 * 3072 * 2 + 3072 * 132
    assert B.workspace_bytes("int4", 4096, 0, 3072) == -1
    assert B.workspace_bytes("int4", 4096, 100, 3072) == -1


FAKE = 1 << 20   # never dereferenced: every call below fails validation first


@pytest.mark.parametrize("args,status", [
    ((0, 64, 100, 32), 2),      # K not a multiple of 256
    ((0, 0, 256, 32), 2),       # M = 0
    ((0, 64, 256, 16), 2),      # unsupported rank
    ((5, 64, 256, 32), 1),      # bad precision
])
def test_quantize_act_validation(args, status):
    prec, M, K, r = args
    s = B.lib.svdq_quantize_act(prec, M, K, r, FAKE, FAKE, FAKE, 1.0, 1.0, FAKE, FAKE, FAKE, None)
    assert s == status, B.lib.svdq_last_error()


def test_quantize_act_null_and_misaligned():
    s = B.lib.svdq_quantize_act(0, 64, 256, 32, None, FAKE, FAKE, 1.0, 1.0, FAKE, FAKE, FAKE, None)
    assert s == 1
    s = B.lib.svdq_quantize_act(0, 64, 256, 32, FAKE + 2, FAKE, FAKE, 1.0, 1.0, FAKE, FAKE, FAKE, None)
    assert s == 1 and b"aligned" in B.lib.svdq_last_error()
    s = B.lib.svdq_quantize_act(0, 64, 256, 32, FAKE, FAKE, FAKE, 0.0, 1.0, FAKE, FAKE, FAKE, None)
    assert s == 1


@pytest.mark.parametrize("M,N,K,status", [(64, 100, 256, 2), (64, 256, 200, 2), (0, 256, 256, 2)])
def test_gemm_validation(M, N, K, status):
    s = B.lib.svdq_w4a4_gemm(0, M, N, K, 32, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, 1.0, FAKE, None, None)
    assert s == status


def test_linear_workspace_too_small():
    s = B.lib.svdq_w4a4_linear(0, 64, 256, 256, 32, FAKE, FAKE, FAKE, 1.0, FAKE, FAKE, 1.0, FAKE, None, FAKE,
                               FAKE, 16, None, None)
    assert s == 1 and b"workspace" in B.lib.svdq_last_error()


def test_awq_validation():
    assert B.lib.awq_w4a16_linear(4, 100, 256, FAKE, FAKE, FAKE, FAKE, None, FAKE, None) == 2
    assert B.lib.awq_w4a16_linear(4, 128, 100, FAKE, FAKE, FAKE, FAKE, None, FAKE, None) == 2
    assert B.lib.awq_w4a16_linear(4, 128, 256, None, FAKE, FAKE, FAKE, None, FAKE, None) == 1


def test_gelu_mlp_sizes():
    # fp32 [M, 32] low-rank sums, rounded up to 256 bytes
    assert B.gelu_quant_work_bytes(4096) == 4096 * 32 * 4
    assert B.gelu_quant_work_bytes(301) == 301 * 128 + (-301 * 128) % 256
    assert B.gelu_quant_work_bytes(0) == -1
    assert B.mlp_workspace_bytes(4096, 3072, 12288) == (B.workspace_bytes("nvfp4", 4096, 12288, 3072) +
                                                         B.workspace_bytes("nvfp4", 4096, 3072, 12288) +
                                                         B.gelu_quant_work_bytes(4096))


@pytest.mark.parametrize("M,N,K,rank,status", [
    (64, 384, 256, 32, 2),      # N (the next layer's K) not a multiple of 256
    (64, 256, 200, 32, 2),      # K not a multiple of 256
    (0, 256, 256, 32, 2),       # M = 0
    (64, 256, 256, 8, 2),       # unsupported rank
])
def test_gemm_gelu_quant_validation(M, N, K, rank, status):
    P = ctypes.c_void_p
    args = [M, N, K, rank] + [P(FAKE)] * 7 + [ctypes.c_float(1.0), P(FAKE), P(FAKE), ctypes.c_float(1.0),
                                               ctypes.c_float(1.0)] + [P(FAKE)] * 4 + [1 << 30, None, None]
    assert B.lib.svdq_w4a4_gemm_gelu_quant(*args) == status


def test_gemm_gelu_quant_rejects_small_work_and_bad_scale():
    P = ctypes.c_void_p
    base = [64, 256, 256, 32] + [P(FAKE)] * 7 + [ctypes.c_float(1.0), P(FAKE), P(FAKE)]
    tail = [P(FAKE)] * 4
    ok_scales = [ctypes.c_float(1.0), ctypes.c_float(1.0)]
    assert B.lib.svdq_w4a4_gemm_gelu_quant(*(base + ok_scales + tail + [16, None, None])) == 1
    assert b"work buffer" in B.lib.svdq_last_error()
    assert B.lib.svdq_w4a4_gemm_gelu_quant(*(base + [ctypes.c_float(0.0), ctypes.c_float(1.0)] + tail +
                                             [1 << 30, None, None])) == 1
    assert b"tensor scales" in B.lib.svdq_last_error()
