"""B200 (sm_100a) SVDQuant W4A4 and AWQ W4A16 linear layers.

Thin ctypes binding over ``lib/libsvdq_b200.so`` (C ABI in ``include/svdq.h``).
Every function here only marshals arguments: it checks dtypes / devices,
allocates outputs with torch when the caller gives none, and passes raw
pointers and the current CUDA stream to the library.  All arithmetic of the
layer happens in the library's CUDA kernels (or, for the offline weight pack,
in its C++ host code).  If the library is missing, importing this package
raises: there is no fallback.
"""
import ctypes
import os

import numpy as np
import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "lib", "libsvdq_b200.so")

SVDQ_NVFP4 = 0
SVDQ_INT4 = 1
SVDQ_RANK = 32
PRECISIONS = {"nvfp4": SVDQ_NVFP4, "int4": SVDQ_INT4}


class SvdqError(RuntimeError):
    def __init__(self, status, message):
        super().__init__(f"svdq status {status}: {message}")
        self.status = status


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"CUDA library not built: {LIB_PATH} is missing "
                          "(run `python bit_w4a4_diffusion_b200/build.py`)")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, F, LL, U = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_longlong, ctypes.c_ulonglong
    sig = {
        "svdq_status_string": (ctypes.c_char_p, [I]),
        "svdq_last_error": (ctypes.c_char_p, []),
        "svdq_version": (I, []),
        "svdq_set_timeout_ns": (None, [U]),
        "svdq_get_timeout_ns": (U, []),
        "svdq_device_status": (I, [P, I, P]),
        "svdq_act_scale_bytes": (LL, [I, I, I]),
        "svdq_weight_scale_bytes": (LL, [I, I, I]),
        "svdq_workspace_bytes": (LL, [I, I, I, I, I]),
        "svdq_workspace_offsets": (I, [I, I, I, I, I, P]),
        "svdq_scales_to_rowmajor": (I, [I, I, P, P]),
        "svdq_scales_from_rowmajor": (I, [I, I, P, P]),
        "svdq_pack_weights": (I, [I, I, I, I, P, P, P, P, P, P, P, P, P, P]),
        "svdq_calibrate": (I, [I, I, I, I, I, I, P, P, P, P, P, P, P]),
        "svdq_quantize_act": (I, [I, I, I, I, P, P, P, F, F, P, P, P, P]),
        "svdq_w4a4_gemm": (I, [I, I, I, I, I, P, P, P, P, P, P, P, F, P, P, P]),
        "svdq_w4a4_linear": (I, [I, I, I, I, I, P, P, P, F, P, P, F, P, P, P, P, LL, P, P]),
        "svdq_gelu_quant_work_bytes": (LL, [I]),
        "svdq_w4a4_gemm_gelu_quant": (I, [I, I, I, I, P, P, P, P, P, P, P, F, P, P, F, F, P, P, P, P, LL, P, P]),
        "svdq_mlp_workspace_bytes": (LL, [I, I, I, I]),
        "svdq_w4a4_mlp_gelu": (I, [I, I, I, I, P, P, P, F, P, P, F, P, P, P, P, F, P, P, F, P, P, P, P, LL, P,
                                   P]),
        "svdq_w4a4_gemm_qkv_norm_rope": (I, [I, I, I, I, P, P, P, P, P, P, P, F, I, I, P, P, P, P, P, P, P]),
        "svdq_w4a4_qkv_norm_rope_linear": (I, [I, I, I, I, I, P, P, P, F, P, P, F, P, P, P, P, P, P, P, P, LL, P,
                                               P]),
        "svdq_noalloc_scratch_bytes": (LL, []),
        "svdq_w4a4_linear_noalloc": (I, [I, I, I, I, I, P, P, P, F, P, P, F, P, P, P, P, P]),
        "awq_pack_weights": (I, [I, I, P, P, P, P]),
        "awq_w4a16_linear": (I, [I, I, I, P, P, P, P, P, P, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = _load()


def _check(status):
    if status != 0:
        msg = lib.svdq_last_error().decode(errors="replace")
        raise SvdqError(status, msg or lib.svdq_status_string(status).decode())


def _prec(precision):
    return PRECISIONS[precision] if isinstance(precision, str) else int(precision)


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, torch.Tensor):
        assert t.is_contiguous(), "tensors must be contiguous"
        return t.data_ptr()
    if isinstance(t, np.ndarray):
        assert t.flags["C_CONTIGUOUS"], "arrays must be C-contiguous"
        return t.ctypes.data
    return int(t)


def _stream(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dev_bf16(t, name):
    if not (isinstance(t, torch.Tensor) and t.is_cuda and t.dtype == torch.bfloat16):
        raise TypeError(f"{name} must be a CUDA bfloat16 tensor")
    return t


# ------------------------------------------------------------------ sizes ---

def act_scale_bytes(precision, M, K):
    return int(lib.svdq_act_scale_bytes(_prec(precision), M, K))


def weight_scale_bytes(precision, N, K):
    return int(lib.svdq_weight_scale_bytes(_prec(precision), N, K))


def workspace_bytes(precision, M, N, K, rank=SVDQ_RANK):
    """Bytes of the workspace of a layer [M, K] -> [M, N].  Its first 64 KiB
    are control words that must be zero before the first call on it
    (allocate it zeroed); every call leaves them zero."""
    return int(lib.svdq_workspace_bytes(_prec(precision), M, N, K, rank))


def workspace_offsets(precision, M, N, K, rank=SVDQ_RANK):
    """Byte offsets in a layer workspace: control words, act codes, act
    scales, lora_act, the precision's own region (NVFP4: the one-kernel
    layer's low-rank partial sums; INT4: the fp16 operands), end."""
    off = np.zeros(6, np.int64)
    _check(lib.svdq_workspace_offsets(_prec(precision), M, N, K, rank, off.ctypes.data))
    return [int(v) for v in off]


def set_timeout_ns(ns):
    lib.svdq_set_timeout_ns(int(ns))


def device_status(clear=True, stream=None):
    """The library's own device status word on the current device: the code
    of a bounded wait that gave up in a call made with ``dev_status=None``
    (0 if none since the last clear).  Waits for ``stream``."""
    v = ctypes.c_int(0)
    _check(lib.svdq_device_status(ctypes.byref(v), 1 if clear else 0, _stream(stream)))
    return int(v.value)


def check_device_status(stream=None):
    """Raise SvdqError(5) if a call made with ``dev_status=None`` timed out on
    the device since the last check (the word is cleared either way)."""
    code = device_status(clear=True, stream=stream)
    if code != 0:
        raise SvdqError(5, f"a device-side wait gave up (code {code}); outputs of the calls since the last "
                           "check are not valid")


def get_timeout_ns():
    return int(lib.svdq_get_timeout_ns())


def scales_to_rowmajor(tiled, rows, K):
    tiled = np.ascontiguousarray(np.asarray(tiled, dtype=np.uint8))
    out = np.empty((rows, K // 16), dtype=np.uint8)
    _check(lib.svdq_scales_to_rowmajor(rows, K, _ptr(tiled), _ptr(out)))
    return out


def scales_from_rowmajor(rowmajor, rows, K):
    rowmajor = np.ascontiguousarray(np.asarray(rowmajor, dtype=np.uint8))
    out = np.empty(weight_scale_bytes(SVDQ_NVFP4, rows, K), dtype=np.uint8)
    _check(lib.svdq_scales_from_rowmajor(rows, K, _ptr(rowmajor), _ptr(out)))
    return out


# ------------------------------------------------------------------ host pack

def svdq_pack_weights(precision, W_bits, smooth, L1_bits, L2_bits, rank=SVDQ_RANK):
    """Host pack.  W_bits uint16 [N,K], smooth fp32 [K], L1_bits uint16 [K,r],
    L2_bits uint16 [r,N].  Returns a dict of host numpy arrays."""
    p = _prec(precision)
    W_bits = np.ascontiguousarray(W_bits, dtype=np.uint16)
    N, K = W_bits.shape
    smooth = np.ascontiguousarray(smooth, dtype=np.float32)
    L1_bits = np.ascontiguousarray(L1_bits, dtype=np.uint16)
    L2_bits = np.ascontiguousarray(L2_bits, dtype=np.uint16)
    out = {
        "codes": np.empty((N, K // 2), np.uint8),
        "scales": np.empty(max(weight_scale_bytes(p, N, K), 1), np.uint8),
        "weight_scale": np.zeros(1, np.float32),
        "inv_smooth": np.empty(K, np.float32),
        "lora_down": np.empty((rank, K), np.uint16),     # bits: fp16 (NVFP4) or bf16 (INT4)
        "lora_up": np.empty((N, 2 * rank), np.uint16),
    }
    _check(lib.svdq_pack_weights(p, N, K, rank, _ptr(W_bits), _ptr(smooth), _ptr(L1_bits), _ptr(L2_bits),
                                 _ptr(out["codes"]), _ptr(out["scales"]), _ptr(out["weight_scale"]),
                                 _ptr(out["inv_smooth"]), _ptr(out["lora_down"]), _ptr(out["lora_up"])))
    if p == SVDQ_NVFP4:
        out["lora_down"] = out["lora_down"].view(np.float16)   # fp16 operand for NVFP4
    out["N"], out["K"], out["rank"], out["precision"] = N, K, rank, p
    return out


def svdq_calibrate(x_bits, W_bits, omega, rank=SVDQ_RANK, power_iters=4):
    """Host calibration: x_bits [M, K], W_bits [N, K] (uint16 bf16 patterns),
    omega [N, rank + p] fp64.  Returns (smooth fp32 [K], L1 bits [K, rank],
    L2 bits [rank, N], act_scale fp32)."""
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    W_bits = np.ascontiguousarray(W_bits, dtype=np.uint16)
    omega = np.ascontiguousarray(omega, dtype=np.float64)
    M, K = x_bits.shape
    N = W_bits.shape[0]
    smooth = np.empty(K, np.float32)
    L1 = np.empty((K, rank), np.uint16)
    L2 = np.empty((rank, N), np.uint16)
    s_a = np.zeros(1, np.float32)
    _check(lib.svdq_calibrate(N, K, M, rank, omega.shape[1] - rank, power_iters, _ptr(W_bits), _ptr(x_bits),
                              _ptr(omega), _ptr(smooth), _ptr(L1), _ptr(L2), _ptr(s_a)))
    return smooth, L1, L2, np.float32(s_a[0])


def awq_pack_weights(W_bits):
    W_bits = np.ascontiguousarray(W_bits, dtype=np.uint16)
    N, K = W_bits.shape
    out = {"qweight": np.empty((N, K // 2), np.uint8), "scales": np.empty((N, K // 64), np.uint16),
           "zeros": np.empty((N, K // 128), np.uint8)}
    _check(lib.awq_pack_weights(N, K, _ptr(W_bits), _ptr(out["qweight"]), _ptr(out["scales"]), _ptr(out["zeros"])))
    out["N"], out["K"] = N, K
    return out


def bits_to_bf16(bits, device=None):
    """uint16 bit patterns (numpy) -> torch bfloat16 tensor (optionally on a device)."""
    t = torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint16).view(np.int16)).view(torch.bfloat16)
    return t.to(device) if device is not None else t


def to_device(packed, device="cuda"):
    """Copy a host pack (dict of numpy arrays) to device tensors."""
    d = {}
    for k, v in packed.items():
        if isinstance(v, np.ndarray):
            if v.dtype == np.uint16:
                d[k] = bits_to_bf16(v, device)
            else:
                d[k] = torch.from_numpy(v).to(device)
        else:
            d[k] = v
    if "weight_scale" in packed:
        d["weight_scale_f"] = float(np.asarray(packed["weight_scale"]).reshape(-1)[0])
    return d


# ------------------------------------------------------------------ device

def svdq_quantize_act(precision, x, inv_smooth, lora_down, act_scale, weight_scale=1.0, out=None, stream=None,
                      rank=SVDQ_RANK):
    p = _prec(precision)
    _dev_bf16(x, "x")
    M, K = x.shape
    if act_scale_bytes(p, M, K) < 0 or M <= 0:
        raise SvdqError(2, f"unsupported shape M={M} K={K}")
    if out is None:
        dev = x.device
        out = (torch.empty((M, K // 2), dtype=torch.uint8, device=dev),
               torch.empty(act_scale_bytes(p, M, K), dtype=torch.uint8, device=dev),
               torch.empty((M, 2 * rank), dtype=torch.bfloat16, device=dev))
    codes, scales, lora_act = out
    _check(lib.svdq_quantize_act(p, M, K, rank, _ptr(x), _ptr(inv_smooth), _ptr(lora_down), float(act_scale),
                                 float(weight_scale), _ptr(codes), _ptr(scales), _ptr(lora_act), _stream(stream)))
    return codes, scales, lora_act


def svdq_w4a4_gemm(precision, act_codes, act_scales, lora_act, w, alpha, bias=None, y=None, dev_status=None,
                   stream=None):
    """w: device dict from to_device(svdq_pack_weights(...))."""
    p = _prec(precision)
    M = act_codes.shape[0]
    N, K, rank = w["N"], w["K"], w["rank"]
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=act_codes.device)
    _check(lib.svdq_w4a4_gemm(p, M, N, K, rank, _ptr(act_codes), _ptr(act_scales), _ptr(lora_act),
                              _ptr(w["codes"]), _ptr(w["scales"]), _ptr(w["lora_up"]), _ptr(bias), float(alpha),
                              _ptr(y), _ptr(dev_status), _stream(stream)))
    return y


def svdq_w4a4_linear(precision, x, w, act_scale, bias=None, y=None, workspace=None, dev_status=None, stream=None):
    p = _prec(precision)
    _dev_bf16(x, "x")
    M, K = x.shape
    N, rank = w["N"], w["rank"]
    assert K == w["K"]
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    if workspace is None:
        workspace = torch.zeros(workspace_bytes(p, M, N, K, rank), dtype=torch.uint8, device=x.device)
    wscale = w["weight_scale_f"]
    _check(lib.svdq_w4a4_linear(p, M, N, K, rank, _ptr(x), _ptr(w["inv_smooth"]), _ptr(w["lora_down"]),
                                float(act_scale), _ptr(w["codes"]), _ptr(w["scales"]), wscale, _ptr(w["lora_up"]),
                                _ptr(bias), _ptr(y), _ptr(workspace), workspace.numel(), _ptr(dev_status),
                                _stream(stream)))
    return y


def svdq_w4a4_linear_noalloc(precision, x, w, act_scale, bias=None, y=None, dev_status=None, stream=None):
    """svdq_w4a4_linear without a workspace: the quantized activations live in
    the library's built-in device scratch (see include/svdq.h)."""
    p = _prec(precision)
    _dev_bf16(x, "x")
    M, K = x.shape
    N, rank = w["N"], w["rank"]
    assert K == w["K"]
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    _check(lib.svdq_w4a4_linear_noalloc(p, M, N, K, rank, _ptr(x), _ptr(w["inv_smooth"]), _ptr(w["lora_down"]),
                                        float(act_scale), _ptr(w["codes"]), _ptr(w["scales"]), w["weight_scale_f"],
                                        _ptr(w["lora_up"]), _ptr(bias), _ptr(y), _ptr(dev_status),
                                        _stream(stream)))
    return y


def gelu_quant_work_bytes(M):
    return int(lib.svdq_gelu_quant_work_bytes(M))


def mlp_workspace_bytes(M, K, N_hidden, rank=SVDQ_RANK):
    return int(lib.svdq_mlp_workspace_bytes(M, K, N_hidden, rank))


def svdq_w4a4_gemm_gelu_quant(act_codes, act_scales, lora_act, w, alpha, w_next, next_act_scale, bias=None,
                              out=None, work=None, dev_status=None, stream=None):
    """The up layer's NVFP4 GEMM with the GELU-MLP epilogue.  w, w_next:
    device dicts of the up layer and of the layer that consumes its GELU
    output.  Returns that layer's (codes, scales, lora_act)."""
    M = act_codes.shape[0]
    N, K, rank = w["N"], w["K"], w["rank"]
    if w_next["K"] != N:
        raise SvdqError(2, f"next layer's K={w_next['K']} differs from N={N}")
    dev = act_codes.device
    if out is None:
        out = (torch.empty((M, N // 2), dtype=torch.uint8, device=dev),
               torch.empty(act_scale_bytes(SVDQ_NVFP4, M, N), dtype=torch.uint8, device=dev),
               torch.empty((M, 2 * rank), dtype=torch.bfloat16, device=dev))
    if work is None:
        work = torch.empty(max(gelu_quant_work_bytes(M), 1), dtype=torch.uint8, device=dev)
    codes, scales, lora = out
    _check(lib.svdq_w4a4_gemm_gelu_quant(M, N, K, rank, _ptr(act_codes), _ptr(act_scales), _ptr(lora_act),
                                         _ptr(w["codes"]), _ptr(w["scales"]), _ptr(w["lora_up"]), _ptr(bias),
                                         float(alpha), _ptr(w_next["inv_smooth"]), _ptr(w_next["lora_down"]),
                                         float(next_act_scale), w_next["weight_scale_f"], _ptr(codes), _ptr(scales),
                                         _ptr(lora), _ptr(work), work.numel(), _ptr(dev_status), _stream(stream)))
    return codes, scales, lora


def svdq_w4a4_mlp_gelu(x, w_up, up_act_scale, w_down, down_act_scale, up_bias=None, down_bias=None, y=None,
                       workspace=None, dev_status=None, stream=None):
    """y = down(GELU(up(x))) with two NVFP4 svdq_w4a4 layers (device dicts)."""
    _dev_bf16(x, "x")
    M, K = x.shape
    N, rank = w_up["N"], w_up["rank"]
    if w_up["K"] != K or w_down["K"] != N or w_down["N"] != K:
        raise SvdqError(2, "layer shapes do not chain: up [K -> N], down [N -> K]")
    if y is None:
        y = torch.empty((M, K), dtype=torch.bfloat16, device=x.device)
    if workspace is None:
        workspace = torch.zeros(max(mlp_workspace_bytes(M, K, N, rank), 1), dtype=torch.uint8, device=x.device)
    _check(lib.svdq_w4a4_mlp_gelu(M, K, N, rank, _ptr(x), _ptr(w_up["inv_smooth"]), _ptr(w_up["lora_down"]),
                                  float(up_act_scale), _ptr(w_up["codes"]), _ptr(w_up["scales"]),
                                  w_up["weight_scale_f"], _ptr(w_up["lora_up"]), _ptr(up_bias),
                                  _ptr(w_down["inv_smooth"]), _ptr(w_down["lora_down"]), float(down_act_scale),
                                  _ptr(w_down["codes"]), _ptr(w_down["scales"]), w_down["weight_scale_f"],
                                  _ptr(w_down["lora_up"]), _ptr(down_bias), _ptr(y), _ptr(workspace),
                                  workspace.numel(), _ptr(dev_status), _stream(stream)))
    return y


def svdq_w4a4_gemm_qkv_norm_rope(act_codes, act_scales, lora_act, w, alpha, heads, gamma_q, gamma_k, rope_cos,
                                 rope_sin, bias=None, y=None, dev_status=None, stream=None, head_dim=128):
    """The fused QKV projection's GEMM with RMSNorm (Q, K heads) and RoPE in
    its epilogue; w: device dict of the [3 * heads * head_dim, K] layer;
    rope_cos / rope_sin: fp32 [head_dim / 2, M] (pair-major)."""
    M = act_codes.shape[0]
    N, K, rank = w["N"], w["K"], w["rank"]
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=act_codes.device)
    _check(lib.svdq_w4a4_gemm_qkv_norm_rope(M, N, K, rank, _ptr(act_codes), _ptr(act_scales), _ptr(lora_act),
                                            _ptr(w["codes"]), _ptr(w["scales"]), _ptr(w["lora_up"]), _ptr(bias),
                                            float(alpha), int(heads), int(head_dim), _ptr(gamma_q), _ptr(gamma_k),
                                            _ptr(rope_cos), _ptr(rope_sin), _ptr(y), _ptr(dev_status),
                                            _stream(stream)))
    return y


def svdq_w4a4_qkv_norm_rope_linear(x, w, act_scale, heads, gamma_q, gamma_k, rope_cos, rope_sin, bias=None, y=None,
                                   workspace=None, dev_status=None, stream=None, head_dim=128):
    _dev_bf16(x, "x")
    M, K = x.shape
    N, rank = w["N"], w["rank"]
    if K != w["K"] or N != 3 * int(heads) * int(head_dim):
        raise SvdqError(2, f"weights [{N}, {w['K']}] do not match x [{M}, {K}] with {heads} heads of {head_dim}")
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    if workspace is None:
        workspace = torch.zeros(workspace_bytes(SVDQ_NVFP4, M, N, K, rank), dtype=torch.uint8, device=x.device)
    _check(lib.svdq_w4a4_qkv_norm_rope_linear(M, K, int(heads), int(head_dim), rank, _ptr(x), _ptr(w["inv_smooth"]),
                                              _ptr(w["lora_down"]), float(act_scale), _ptr(w["codes"]),
                                              _ptr(w["scales"]), w["weight_scale_f"], _ptr(w["lora_up"]), _ptr(bias),
                                              _ptr(gamma_q), _ptr(gamma_k), _ptr(rope_cos), _ptr(rope_sin), _ptr(y),
                                              _ptr(workspace), workspace.numel(), _ptr(dev_status), _stream(stream)))
    return y


def awq_w4a16_linear(x, w, bias=None, y=None, stream=None):
    _dev_bf16(x, "x")
    M, K = x.shape
    N = w["N"]
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    _check(lib.awq_w4a16_linear(M, N, K, _ptr(x), _ptr(w["qweight"]), _ptr(w["scales"]), _ptr(w["zeros"]),
                                _ptr(bias), _ptr(y), _stream(stream)))
    return y
