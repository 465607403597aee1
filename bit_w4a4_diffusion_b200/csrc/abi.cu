// C-ABI entry points (declared in include/svdq.h): argument checks, device
// checks, tensor-map set-up and kernel launches.  No allocation happens here:
// every buffer belongs to the caller.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cmath>
#include <cstring>
#include <algorithm>
#include <atomic>
#include <mutex>

#include "svdq.h"
#include "svdq_internal.h"

using namespace svdq;

namespace {

thread_local char g_last_error[512] = "";

int fail(int status, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return status;
}

struct DeviceInfo {
  bool checked = false;
  bool ok = false;
  int sms = 0;
  int cc_major = 0, cc_minor = 0;
};
constexpr int kMaxDevices = 64;
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

// Returns SVDQ_OK and the SM count if the current device is an sm_100 part.
int check_device(int* sms) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(SVDQ_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return fail(SVDQ_ERR_UNSUPPORTED_DEVICE, "device index %d", dev);
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.checked) {
    cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&d.cc_minor, cudaDevAttrComputeCapabilityMinor, dev);
    cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
    d.ok = (d.cc_major == 10 && d.cc_minor == 0);
    d.checked = true;
  }
  if (!d.ok)
    return fail(SVDQ_ERR_UNSUPPORTED_DEVICE, "this library is built for sm_100a (B200); device %d is sm_%d%d", dev,
                d.cc_major, d.cc_minor);
  *sms = d.sms;
  return SVDQ_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

int64_t round_up(int64_t a, int64_t b) { return (a + b - 1) / b * b; }

std::atomic<unsigned long long> g_timeout_ns{1000000000ull};
unsigned long long svdq_timeout_ns() { return g_timeout_ns.load(std::memory_order_relaxed); }

// Programmatic dependent launch for every kernel unless SVDQ_PDL=0 (read at
// every call, so a process can compare the two).
bool pdl_on() {
  const char* v = getenv("SVDQ_PDL");
  return !(v && strcmp(v, "0") == 0);
}

int check_cuda(cudaError_t e, const char* what) {
  if (e != cudaSuccess) return fail(SVDQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return SVDQ_OK;
}

// The library's own device status word: every launch whose caller passes no
// dev_status reports a wait that gave up here, so that such a call is never
// mistaken for a good one; svdq_device_status() reads and clears it.  A
// file-scope device variable exists once in each context that loads this
// module.
__device__ int g_lib_status;

struct SymbolSlot {
  unsigned long long ctx_id = 0;
  void* ptr = nullptr;
};
SymbolSlot g_status_slot[kMaxDevices];
std::mutex g_status_mu;

// Device address of g_lib_status in the current context.
int lib_status_word(int** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(SVDQ_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return fail(SVDQ_ERR_UNSUPPORTED_DEVICE, "device index %d", dev);
  const unsigned long long ctx = svdq::current_context_id();
  std::lock_guard<std::mutex> lk(g_status_mu);
  SymbolSlot& s = g_status_slot[dev];
  if (s.ptr == nullptr || ctx == 0 || s.ctx_id != ctx) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_lib_status);
    if (e != cudaSuccess || p == nullptr)
      return fail(SVDQ_ERR_CUDA, "cudaGetSymbolAddress(status word): %s", cudaGetErrorString(e));
    s.ptr = p;
    s.ctx_id = ctx;
  }
  *out = static_cast<int*>(s.ptr);
  return SVDQ_OK;
}

// The caller's status word, or the library's when the caller gives none.
int resolve_status(int** dev_status) {
  if (*dev_status != nullptr) return SVDQ_OK;
  return lib_status_word(dev_status);
}

// Units per 128-row block of the fused layer kernel: the largest divisor of
// K / 256 up to 12 (each unit quantizes K / splits columns).
int fused_splits(int K) {
  const int kb = K / 256;
  for (int sp = 12; sp > 1; --sp)
    if (kb % sp == 0) return sp;
  return 1;
}

}  // namespace

namespace svdq {

int record_error(int status, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return status;
}

unsigned long long current_context_id() {
  using CtxGetCurrentFn = CUresult (*)(CUcontext*);
  using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  if (!get_current || !get_id) return 0;
  CUcontext c = nullptr;
  if (get_current(&c) != CUDA_SUCCESS || c == nullptr) return 0;
  unsigned long long id = 0;
  if (get_id(c, &id) != CUDA_SUCCESS) return 0;
  return id;
}

bool encode_tmap_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
                    uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace svdq

extern "C" {

const char* svdq_status_string(int status) {
  switch (status) {
    case SVDQ_OK: return "ok";
    case SVDQ_ERR_INVALID_ARG: return "invalid argument";
    case SVDQ_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case SVDQ_ERR_UNSUPPORTED_DEVICE: return "unsupported device";
    case SVDQ_ERR_CUDA: return "CUDA error";
    case SVDQ_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    default: return "unknown status";
  }
}

const char* svdq_last_error(void) { return g_last_error; }

int svdq_version(void) { return SVDQ_VERSION; }

void svdq_set_timeout_ns(unsigned long long ns) { g_timeout_ns.store(ns, std::memory_order_relaxed); }
unsigned long long svdq_get_timeout_ns(void) { return g_timeout_ns.load(std::memory_order_relaxed); }

int svdq_device_status(int* value, int clear, void* stream) {
  if (!value) return fail(SVDQ_ERR_INVALID_ARG, "null value pointer");
  int sms = 0;
  if (int s = check_device(&sms)) return s;
  int* word = nullptr;
  if (int s = lib_status_word(&word)) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int host = 0;
  if (int s = check_cuda(cudaMemcpyAsync(&host, word, sizeof(int), cudaMemcpyDeviceToHost, st), "status read"))
    return s;
  if (int s = check_cuda(cudaStreamSynchronize(st), "status read")) return s;
  if (clear && host != 0) {
    if (int s = check_cuda(cudaMemsetAsync(word, 0, sizeof(int), st), "status clear")) return s;
    if (int s = check_cuda(cudaStreamSynchronize(st), "status clear")) return s;
  }
  *value = host;
  return SVDQ_OK;
}

long long svdq_act_scale_bytes(int precision, int M, int K) {
  if (M < 0 || K <= 0) return -1;
  const int64_t mp = round_up(M > 0 ? M : 1, 256);
  if (precision == SVDQ_NVFP4) return (K % 64) ? -1 : mp * (K / 16);
  if (precision == SVDQ_INT4) return (K % 64) ? -1 : mp * (K / 64) * 2;
  return -1;
}

long long svdq_weight_scale_bytes(int precision, int N, int K) { return svdq_act_scale_bytes(precision, N, K); }

// The INT4 layer's fp16-operand region (workspace offset [4]), in bytes from
// its start: A' [M, K] fp16, the scaled lora_act [M, 64] bf16, f_a [M] fp32,
// W' [N, K] fp16, the scaled lora_up [N, 64] bf16, f_w [N] fp32, each
// 256-byte aligned; o[6] is the region's size.
static void int4_operand_offsets(int M, int N, int K, long long (&o)[7]) {
  o[0] = 0;
  o[1] = o[0] + round_up((int64_t)M * K * 2, 256);
  o[2] = o[1] + round_up((int64_t)M * 64 * 2, 256);
  o[3] = o[2] + round_up((int64_t)M * 4, 256);
  o[4] = o[3] + round_up((int64_t)N * K * 2, 256);
  o[5] = o[4] + round_up((int64_t)N * 64 * 2, 256);
  o[6] = o[5] + round_up((int64_t)N * 4, 256);
}

int svdq_workspace_offsets(int precision, int M, int N, int K, int rank, long long* offsets) {
  if (!offsets) return fail(SVDQ_ERR_INVALID_ARG, "null offsets");
  if (precision != SVDQ_NVFP4 && precision != SVDQ_INT4)
    return fail(SVDQ_ERR_INVALID_ARG, "precision %d is not SVDQ_NVFP4 or SVDQ_INT4", precision);
  if (M <= 0 || K <= 0 || K % 256 != 0 || rank != SVDQ_RANK)
    return fail(SVDQ_ERR_UNSUPPORTED_SHAPE, "M=%d K=%d rank=%d", M, K, rank);
  if (N < 0 || (precision == SVDQ_INT4 && (N == 0 || N % 128 != 0)))
    return fail(SVDQ_ERR_UNSUPPORTED_SHAPE, "N=%d (INT4 needs a positive multiple of 128)", N);
  const long long codes = kSyncBytes;
  const long long scales = codes + round_up((int64_t)M * (K / 2), 256);
  const long long lora = scales + round_up(svdq_act_scale_bytes(precision, M, K), 256);
  const long long upart = lora + round_up((int64_t)M * 2 * rank * 2, 256);
  long long int4_region[7];
  int4_operand_offsets(M, N, K, int4_region);
  const long long end =
      upart + (precision == SVDQ_NVFP4 ? round_up((int64_t)fused_splits(K) * round_up(M, 256) * 32 * 4, 256)
                                       : int4_region[6]);
  offsets[0] = 0;
  offsets[1] = codes;
  offsets[2] = scales;
  offsets[3] = lora;
  offsets[4] = upart;
  offsets[5] = end;
  return SVDQ_OK;
}

long long svdq_workspace_bytes(int precision, int M, int N, int K, int rank) {
  long long off[6];
  if (svdq_workspace_offsets(precision, M, N, K, rank, off) != SVDQ_OK) return -1;
  return off[5];
}

// NVFP4 activation quantizer: the TMA-fed kernel unless
// SVDQ_NVFP4_QUANT_KERNEL=copy asks for the per-thread-copy kernel (read at
// every call).  Both give bit-identical codes and scales; the low-rank
// activations differ only by the order of their fp32 partial sums.
static bool use_copy_quantizer() {
  const char* v = getenv("SVDQ_NVFP4_QUANT_KERNEL");
  return v && strcmp(v, "copy") == 0;
}

// w_side (INT4 only, or null): the layer's weight rows to convert to fp16
// operands in extra blocks of the quantizer's launch (int4_dequant_rows.cuh).
static int quantize_act_impl(int precision, int M, int K, int rank, const void* x, const float* inv_smooth,
                             const void* lora_down, float act_scale, float weight_scale, void* act_codes,
                             void* act_scales, void* lora_act, int* dev_status, void* stream,
                             const DequantInt4Params* w_side = nullptr) {
  if (precision != SVDQ_NVFP4 && precision != SVDQ_INT4)
    return fail(SVDQ_ERR_INVALID_ARG, "precision %d is not SVDQ_NVFP4 or SVDQ_INT4", precision);
  if (M <= 0 || K <= 0) return fail(SVDQ_ERR_UNSUPPORTED_SHAPE, "M=%d K=%d must be positive", M, K);
  if (K % 256 != 0) return fail(SVDQ_ERR_UNSUPPORTED_SHAPE, "K=%d must be a multiple of 256", K);
  if (rank != SVDQ_RANK) return fail(SVDQ_ERR_UNSUPPORTED_SHAPE, "rank=%d; this build supports rank %d", rank, SVDQ_RANK);
  if (!x || !inv_smooth || !lora_down || !act_codes || !act_scales || !lora_act)
    return fail(SVDQ_ERR_INVALID_ARG, "null pointer argument");
  if (!aligned16(x) || !aligned16(inv_smooth) || !aligned16(lora_down) || !aligned16(act_codes) ||
      !aligned16(lora_act) || !aligned16(act_scales))
    return fail(SVDQ_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  // Scales from 2^-100 up keep every block reciprocal 1/(E4M3 * s) finite in fp32.
  if (precision == SVDQ_NVFP4 && !(act_scale >= 0x1p-100f && weight_scale >= 0x1p-100f &&
                                   act_scale < 0x1p100f && weight_scale < 0x1p100f))
    return fail(SVDQ_ERR_INVALID_ARG, "NVFP4 tensor scales must lie in [2^-100, 2^100) (act %g, weight %g)",
                act_scale, weight_scale);
  int sms = 0;
  if (int s = check_device(&sms)) return s;
  if (int s = resolve_status(&dev_status)) return s;
  QuantActParams p{};
  p.M = M;
  p.K = K;
  p.M_pad = (int)round_up(M, 256);
  p.x = static_cast<const uint16_t*>(x);
  p.inv_smooth = inv_smooth;
  p.lora_down = static_cast<const uint16_t*>(lora_down);
  p.act_scale = act_scale;
  if (precision == SVDQ_NVFP4) {
    // x_hat enters the fp16 down-projection as x_hat * 2^-e, with 2^e the power
    // of two that maps the calibrated range 2688 s_a into [2^12, 2^13).
    int ex = 0;
    frexpf(2688.0f * act_scale, &ex);  // 2688 s_a = m * 2^ex, m in [0.5, 1)
    const int e = ex - 1 - 12;
    p.lr_in_scale = ldexpf(1.0f, -e);
    p.lora_scale = ldexpf(1.0f, e) / (act_scale * weight_scale);
  } else {
    p.lr_in_scale = 1.0f;
    p.lora_scale = 1.0f;
  }
  p.act_codes = static_cast<uint8_t*>(act_codes);
  p.act_scales = static_cast<uint8_t*>(act_scales);
  p.lora_act = static_cast<uint16_t*>(lora_act);
  p.s1_blocks = p.M_pad / 16;
  if (w_side != nullptr && precision == SVDQ_INT4 && w_side->R > 0) {
    // One conversion block per 32 weight rows (the caller checked that they
    // fit beside the quantizer's own CTAs, two of which fit per SM).
    p.w_side = *w_side;
    p.w_blocks = (w_side->R + 31) / 32;
  }
  if (precision == SVDQ_NVFP4 && !use_copy_quantizer()) {
    // TMA-fed kernel: x [M, K] bf16 and L1^T [32, K] fp16 in 64 x 32 boxes.
    CUtensorMap tx, tl;
    bool ok = encode_tmap_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, K, M, (uint64_t)K * 2, 64, 32,
                             CU_TENSOR_MAP_SWIZZLE_128B);
    ok &= encode_tmap_2d(&tl, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, lora_down, K, SVDQ_RANK, (uint64_t)K * 2, 64, 32,
                         CU_TENSOR_MAP_SWIZZLE_128B);
    if (!ok) return fail(SVDQ_ERR_CUDA, "cuTensorMapEncodeTiled failed for the quantize kernel");
    return check_cuda(launch_quantize_nvfp4(p, tx, tl, dev_status, svdq_timeout_ns(), static_cast<cudaStream_t>(stream), pdl_on()),
                      "quantize_nvfp4 launch");
  }
  return check_cuda(launch_quantize_act(p, precision == SVDQ_NVFP4, static_cast<cudaStream_t>(stream), pdl_on()),
                    "quantize_act launch");
}

int svdq_quantize_act(int precision, int M, int K, int rank, const void* x, const float* inv_smooth,
                      const void* lora_down, float act_scale, float weight_scale, void* act_codes, void* act_scales,
                      void* lora_act, void* stream) {
  return quantize_act_impl(precision, M, K, rank, x, inv_smooth, lora_down, act_scale, weight_scale, act_codes,
                           act_scales, lora_act, nullptr, stream);
}

// NVFP4 GEMM kernel per epilogue kind.  SVDQ_NVFP4_GEMM_KERNEL=pair or
// =single (read at every call, so a process can compare them) forces the
// CTA-pair kernel (256 x 256 tiles on two SMs) or the one-CTA-per-tile
// kernel for every kind; both give bit-identical results (up to the order of
// the GELU-MLP epilogue's atomic low-rank sums).  By default the pair kernel
// runs the plain and QKV epilogues: it streams 38 KB of operands per SM and K
// slice instead of 54 and keeps one block-scale buffer per stage, 14-26%
// faster on the DiT layer shapes and 10% on the fused QKV projection.  The
// GELU-MLP epilogue stays on the single-CTA kernel: it is bound by its own
// arithmetic, which the pair's faster main loop does not shorten, and the
// pair's single accumulator makes it 4% slower there.
static bool use_pair_gemm(bool gelu) {
  const char* v = getenv("SVDQ_NVFP4_GEMM_KERNEL");
  if (v && strcmp(v, "single") == 0) return false;
  if (v && strcmp(v, "pair") == 0) return true;
  return !gelu;
}

// gq != nullptr selects the GELU-MLP epilogue, qk != nullptr the QKV +
// RMSNorm + RoPE epilogue (single-CTA kernel; y's tensor map unused).
static int gemm_nvfp4_impl(int M, int N, int K, const void* act_codes, const void* act_scales, const void* lora_act,
                           const void* w_codes, const void* w_scales, const void* lora_up, const void* bias,
                           float alpha, void* y, int* dev_status, cudaStream_t stream, bool pdl, int sms,
                           const GeluQuantParams* gq = nullptr, const QkvParams* qk = nullptr) {
  GemmTmaps t;
  bool ok = true;
  ok &= encode_tmap_2d(&t.a, CU_TENSOR_MAP_DATA_TYPE_UINT8, act_codes, K / 2, M, K / 2, 128, 128,
                       CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= encode_tmap_2d(&t.b, CU_TENSOR_MAP_DATA_TYPE_UINT8, w_codes, K / 2, N, K / 2, 128, 256,
                       CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= encode_tmap_2d(&t.la, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, lora_act, 2 * SVDQ_RANK, M, 2 * SVDQ_RANK * 2, 64,
                       128, CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= encode_tmap_2d(&t.lb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, lora_up, 2 * SVDQ_RANK, N, 2 * SVDQ_RANK * 2, 64,
                       256, CU_TENSOR_MAP_SWIZZLE_128B);
  if (gq == nullptr && qk == nullptr)
    ok &= encode_tmap_2d(&t.y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, y, N, M, (uint64_t)N * 2, 16, 32,
                         CU_TENSOR_MAP_SWIZZLE_32B);
  else
    t.y = t.a;  // not read by the GELU-MLP epilogue
  if (!ok) return fail(SVDQ_ERR_CUDA, "cuTensorMapEncodeTiled failed (driver entry point unavailable?)");
  GemmNvfp4Params p{};
  p.M = M;
  p.N = N;
  p.K = K;
  p.act_scales = static_cast<const uint8_t*>(act_scales);
  p.w_scales = static_cast<const uint8_t*>(w_scales);
  p.bias = static_cast<const uint16_t*>(bias);
  p.alpha = alpha;
  p.dev_status = dev_status;
  p.timeout_ns = svdq_timeout_ns();
  if (gq != nullptr) p.gq = *gq;
  if (qk != nullptr) p.qk = *qk;
  if (use_pair_gemm(gq != nullptr)) {
    // CTA-pair kernel: half-tile boxes for B and [L2^T|L2^T], and the block
    // scales as 2D maps of 256-byte rows (8 rows = one 2 KB chunk group).
    GemmPairTmaps u;
    u.a = t.a;
    u.la = t.la;
    u.y = t.y;
    const uint64_t sfa_rows = (uint64_t)round_up(M, 256) * (K / 16) / 256;
    const uint64_t sfb_rows = (uint64_t)round_up(N, 256) * (K / 16) / 256;
    ok &= encode_tmap_2d(&u.b, CU_TENSOR_MAP_DATA_TYPE_UINT8, w_codes, K / 2, N, K / 2, 128, 128,
                         CU_TENSOR_MAP_SWIZZLE_128B);
    ok &= encode_tmap_2d(&u.lb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, lora_up, 2 * SVDQ_RANK, N, 2 * SVDQ_RANK * 2, 64,
                         128, CU_TENSOR_MAP_SWIZZLE_128B);
    ok &= encode_tmap_2d(&u.sfa, CU_TENSOR_MAP_DATA_TYPE_UINT8, act_scales, 256, sfa_rows, 256, 256, 8,
                         CU_TENSOR_MAP_SWIZZLE_NONE);
    ok &= encode_tmap_2d(&u.sfb, CU_TENSOR_MAP_DATA_TYPE_UINT8, w_scales, 256, sfb_rows, 256, 256, 8,
                         CU_TENSOR_MAP_SWIZZLE_NONE);
    if (!ok) return fail(SVDQ_ERR_CUDA, "cuTensorMapEncodeTiled failed for the CTA-pair GEMM");
    if (gq != nullptr)
      return check_cuda(launch_gemm_nvfp4_pair_gelu(p, u, stream, pdl), "gemm_nvfp4_pair (GELU-MLP epilogue) launch");
    if (qk != nullptr)
      return check_cuda(launch_gemm_nvfp4_pair_qkv(p, u, stream, pdl), "gemm_nvfp4_pair (QKV epilogue) launch");
    return check_cuda(launch_gemm_nvfp4_pair(p, u, stream, pdl), "gemm_nvfp4_pair launch");
  }
  if (gq != nullptr)
    return check_cuda(launch_gemm_nvfp4_gelu(p, t, sms, stream, pdl), "gemm_nvfp4 (GELU-MLP epilogue) launch");
  if (qk != nullptr)
    return check_cuda(launch_gemm_nvfp4_qkv(p, t, sms, stream, pdl), "gemm_nvfp4 (QKV epilogue) launch");
  return check_cuda(launch_gemm_nvfp4(p, t, sms, stream, pdl), "gemm_nvfp4 launch");
}

static int check_gemm_args(int precision, int M, int N, int K, int rank) {
  if (precision != SVDQ_NVFP4 && precision != SVDQ_INT4)
    return fail(SVDQ_ERR_INVALID_ARG, "precision %d is not SVDQ_NVFP4 or SVDQ_INT4", precision);
  if (M <= 0 || N <= 0 || K <= 0) return fail(SVDQ_ERR_UNSUPPORTED_SHAPE, "M=%d N=%d K=%d must be positive", M, N, K);
  if (K % 256 != 0) return fail(SVDQ_ERR_UNSUPPORTED_SHAPE, "K=%d must be a multiple of 256", K);
  if (N % 128 != 0) return fail(SVDQ_ERR_UNSUPPORTED_SHAPE, "N=%d must be a multiple of 128", N);
  if (rank != SVDQ_RANK) return fail(SVDQ_ERR_UNSUPPORTED_SHAPE, "rank=%d; this build supports rank %d", rank, SVDQ_RANK);
  return SVDQ_OK;
}

static int gemm_int4_impl(int M, int N, int K, const void* act_codes, const void* act_scales, const void* lora_act,
                          const void* w_codes, const void* w_scales, const void* lora_up, const void* bias, void* y,
                          int* dev_status, cudaStream_t stream, bool pdl, int sms) {
  GemmInt4Tmaps t;
  bool ok = true;
  ok &= encode_tmap_2d(&t.a, CU_TENSOR_MAP_DATA_TYPE_UINT8, act_codes, K / 2, M, K / 2, 64, 128,
                       CU_TENSOR_MAP_SWIZZLE_NONE);
  ok &= encode_tmap_2d(&t.b, CU_TENSOR_MAP_DATA_TYPE_UINT8, w_codes, K / 2, N, K / 2, 64, 128,
                       CU_TENSOR_MAP_SWIZZLE_NONE);
  ok &= encode_tmap_2d(&t.la, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, lora_act, 2 * SVDQ_RANK, M, 2 * SVDQ_RANK * 2, 64,
                       128, CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= encode_tmap_2d(&t.lb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, lora_up, 2 * SVDQ_RANK, N, 2 * SVDQ_RANK * 2, 64,
                       128, CU_TENSOR_MAP_SWIZZLE_128B);
  if (!ok) return fail(SVDQ_ERR_CUDA, "cuTensorMapEncodeTiled failed (driver entry point unavailable?)");
  GemmInt4Params p{};
  p.M = M;
  p.N = N;
  p.K = K;
  p.M_pad = (int)round_up(M, 256);
  p.N_pad = (int)round_up(N, 256);
  p.act_scales = static_cast<const uint16_t*>(act_scales);
  p.w_scales = static_cast<const uint16_t*>(w_scales);
  p.bias = static_cast<const uint16_t*>(bias);
  p.y = static_cast<uint16_t*>(y);
  p.dev_status = dev_status;
  p.timeout_ns = svdq_timeout_ns();
  return check_cuda(launch_gemm_int4(p, t, sms, stream, pdl), "gemm_int4 launch");
}

// The INT4 layer's product on the fp16 tensor pipe, from exact fp16 values of
// both operands (dequant_int4.cu).  By default both operands are written out
// in fp16 to the workspace region first (one launch for both), then the NVFP4
// pair kernel runs its fp16 path.  SVDQ_INT4_LAYER_GEMM (read at every call)
// selects instead "dq": the CTA-pair kernel of gemm_int4_pair.cu, which
// builds the fp16 operand tiles itself in shared memory, slice by slice, from
// the codes (the same values and MMAs, so the same y bit for bit; slower on
// B200: 229 against 105 us at M = 4096, K = N = 3072); or "i8":
// svdq_w4a4_gemm's kernel (gemm_int4.cu, which needs no scratch).  All sum
// the same exact products in fp32.
enum class Int4LayerGemm { kF16Operands, kDequantInGemm, kI8 };
static Int4LayerGemm int4_layer_gemm() {
  const char* v = getenv("SVDQ_INT4_LAYER_GEMM");
  if (v && strcmp(v, "i8") == 0) return Int4LayerGemm::kI8;
  if (v && strcmp(v, "dq") == 0) return Int4LayerGemm::kDequantInGemm;
  return Int4LayerGemm::kF16Operands;
}

static int gemm_int4_f16_impl(int M, int N, int K, const void* act_codes, const void* act_scales,
                              const void* lora_act, const void* w_codes, const void* w_scales, const void* lora_up,
                              const void* bias, void* y, uint8_t* region, int* dev_status, cudaStream_t stream,
                              bool pdl, bool in_gemm, bool weights_done = false) {
  long long o[7];
  int4_operand_offsets(M, N, K, o);
  uint16_t* a16 = reinterpret_cast<uint16_t*>(region + o[0]);
  uint16_t* la = reinterpret_cast<uint16_t*>(region + o[1]);
  float* fa = reinterpret_cast<float*>(region + o[2]);
  uint16_t* w16 = reinterpret_cast<uint16_t*>(region + o[3]);
  uint16_t* lb = reinterpret_cast<uint16_t*>(region + o[4]);
  float* fw = reinterpret_cast<float*>(region + o[5]);
  if (in_gemm) {
    // The rows' powers of two and the scaled low-rank operands only; the GEMM
    // builds the fp16 operand tiles from the codes.
    GemmInt4DqTmaps t;
    bool ok = true;
    ok &= encode_tmap_2d(&t.a4, CU_TENSOR_MAP_DATA_TYPE_UINT8, act_codes, K / 2, M, K / 2, 32, 128,
                         CU_TENSOR_MAP_SWIZZLE_NONE);
    ok &= encode_tmap_2d(&t.b4, CU_TENSOR_MAP_DATA_TYPE_UINT8, w_codes, K / 2, N, K / 2, 32, 128,
                         CU_TENSOR_MAP_SWIZZLE_NONE);
    ok &= encode_tmap_2d(&t.la, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, la, 2 * SVDQ_RANK, M, 2 * SVDQ_RANK * 2, 64, 128,
                         CU_TENSOR_MAP_SWIZZLE_128B);
    ok &= encode_tmap_2d(&t.lb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, lb, 2 * SVDQ_RANK, N, 2 * SVDQ_RANK * 2, 64, 128,
                         CU_TENSOR_MAP_SWIZZLE_128B);
    ok &= encode_tmap_2d(&t.y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, y, N, M, (uint64_t)N * 2, 16, 32,
                         CU_TENSOR_MAP_SWIZZLE_32B);
    if (!ok) return fail(SVDQ_ERR_CUDA, "cuTensorMapEncodeTiled failed for the INT4 pair GEMM");
    DequantInt4Params fw_p{N, K, (int)round_up(N, 256), static_cast<const uint8_t*>(w_codes),
                           static_cast<const uint16_t*>(w_scales), static_cast<const uint16_t*>(lora_up), nullptr, lb,
                           fw};
    DequantInt4Params fa_p{M, K, (int)round_up(M, 256), static_cast<const uint8_t*>(act_codes),
                           static_cast<const uint16_t*>(act_scales), static_cast<const uint16_t*>(lora_act), nullptr,
                           la, fa};
    if (int s = check_cuda(launch_dequant_int4(fw_p, fa_p, stream, pdl), "INT4 row factors launch")) return s;
    GemmInt4DqParams q{};
    q.M = M;
    q.N = N;
    q.K = K;
    q.M_pad = (int)round_up(M, 256);
    q.N_pad = (int)round_up(N, 256);
    q.act_scales = static_cast<const uint16_t*>(act_scales);
    q.w_scales = static_cast<const uint16_t*>(w_scales);
    q.bias = static_cast<const uint16_t*>(bias);
    q.row_factor = fa;
    q.col_factor = fw;
    q.dev_status = dev_status;
    q.timeout_ns = svdq_timeout_ns();
    return check_cuda(launch_gemm_int4_pair(q, t, stream, pdl), "gemm_int4_pair launch");
  }
  GemmPairTmaps u;
  bool ok = true;
  ok &= encode_tmap_2d(&u.a, CU_TENSOR_MAP_DATA_TYPE_UINT8, a16, (uint64_t)K * 2, M, (uint64_t)K * 2, 128, 128,
                       CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= encode_tmap_2d(&u.b, CU_TENSOR_MAP_DATA_TYPE_UINT8, w16, (uint64_t)K * 2, N, (uint64_t)K * 2, 128, 128,
                       CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= encode_tmap_2d(&u.la, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, la, 2 * SVDQ_RANK, M, 2 * SVDQ_RANK * 2, 64, 128,
                       CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= encode_tmap_2d(&u.lb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, lb, 2 * SVDQ_RANK, N, 2 * SVDQ_RANK * 2, 64, 128,
                       CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= encode_tmap_2d(&u.y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, y, N, M, (uint64_t)N * 2, 16, 32,
                       CU_TENSOR_MAP_SWIZZLE_32B);
  if (!ok) return fail(SVDQ_ERR_CUDA, "cuTensorMapEncodeTiled failed for the fp16-operand INT4 GEMM");
  u.sfa = u.a;   // not read
  u.sfb = u.a;
  // The weight side is converted here unless the quantizer's launch already
  // did it (int4_w_side): then this launch covers the activation rows only.
  DequantInt4Params da{M, K, (int)round_up(M, 256), static_cast<const uint8_t*>(act_codes),
                       static_cast<const uint16_t*>(act_scales), static_cast<const uint16_t*>(lora_act), a16, la, fa};
  DequantInt4Params dw{weights_done ? 0 : N, K, (int)round_up(N, 256), static_cast<const uint8_t*>(w_codes),
                       static_cast<const uint16_t*>(w_scales), static_cast<const uint16_t*>(lora_up), w16, lb, fw};
  if (int s = check_cuda(launch_dequant_int4(dw, da, stream, pdl), "dequant_int4 launch")) return s;
  GemmNvfp4Params p{};
  p.M = M;
  p.N = N;
  p.K = K;
  p.bias = static_cast<const uint16_t*>(bias);
  p.alpha = 1.0f;
  p.dev_status = dev_status;
  p.timeout_ns = svdq_timeout_ns();
  p.row_factor = fa;
  p.col_factor = fw;
  return check_cuda(launch_gemm_f16_pair(p, u, stream, pdl), "gemm_f16_pair (INT4) launch");
}

int svdq_w4a4_gemm(int precision, int M, int N, int K, int rank, const void* act_codes, const void* act_scales,
                   const void* lora_act, const void* w_codes, const void* w_scales, const void* lora_up,
                   const void* bias, float alpha, void* y, int* dev_status, void* stream) {
  if (int s = check_gemm_args(precision, M, N, K, rank)) return s;
  if (!act_codes || !act_scales || !lora_act || !w_codes || !w_scales || !lora_up || !y)
    return fail(SVDQ_ERR_INVALID_ARG, "null pointer argument");
  if (!aligned16(act_codes) || !aligned16(act_scales) || !aligned16(lora_act) || !aligned16(w_codes) ||
      !aligned16(w_scales) || !aligned16(lora_up) || !aligned16(y) || (bias && !aligned16(bias)))
    return fail(SVDQ_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  if (precision == SVDQ_NVFP4 && !(alpha > 0.f)) return fail(SVDQ_ERR_INVALID_ARG, "alpha must be positive");
  int sms = 0;
  if (int s = check_device(&sms)) return s;
  if (int s = resolve_status(&dev_status)) return s;
  if (precision == SVDQ_INT4)
    return gemm_int4_impl(M, N, K, act_codes, act_scales, lora_act, w_codes, w_scales, lora_up, bias, y, dev_status,
                          static_cast<cudaStream_t>(stream), pdl_on(), sms);
  return gemm_nvfp4_impl(M, N, K, act_codes, act_scales, lora_act, w_codes, w_scales, lora_up, bias, alpha, y,
                         dev_status, static_cast<cudaStream_t>(stream), pdl_on(), sms);
}

static bool nvfp4_scale_ok(float s);

// The NVFP4 layer runs as the quantize kernel followed by the GEMM unless
// SVDQ_LAYER_KERNEL=fused asks for the one-kernel layer (quantizer units
// inside the CTA-pair GEMM; read at every call), which also needs the pair
// GEMM and M within the control region's row blocks.  Measured on B200 at
// the DiT MLP up-projection (4096 x 3072 -> 12288): 96 us one kernel against
// 81.5 us for the two kernels, whose GEMM alone takes 72 us: the quantizer's
// arithmetic (about 14 instructions per element) takes issue slots from the
// GEMM's MMA warp.
static bool use_layer_kernel(int M) {
  const char* v = getenv("SVDQ_LAYER_KERNEL");
  if (!(v && strcmp(v, "fused") == 0)) return false;
  if (!use_pair_gemm(false)) return false;
  return round_up(M, 256) / 128 <= kSyncMaxRowBlocks;
}

// x's quantized form is produced inside the GEMM kernel, in the workspace.
static int layer_nvfp4_impl(int M, int N, int K, const void* x, const float* inv_smooth, const void* lora_down,
                            float act_scale, const void* w_codes, const void* w_scales, float weight_scale,
                            const void* lora_up, const void* bias, void* y, uint8_t* ws, const long long* off,
                            int* dev_status, cudaStream_t stream, bool pdl) {
  uint8_t* codes = ws + off[1];
  uint8_t* scales = ws + off[2];
  uint8_t* lora = ws + off[3];
  GemmPairTmaps u;
  CUtensorMap tx, tl;
  const uint64_t sfa_rows = (uint64_t)round_up(M, 256) * (K / 16) / 256;
  const uint64_t sfb_rows = (uint64_t)round_up(N, 256) * (K / 16) / 256;
  bool ok = true;
  ok &= encode_tmap_2d(&u.a, CU_TENSOR_MAP_DATA_TYPE_UINT8, codes, K / 2, M, K / 2, 128, 128,
                       CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= encode_tmap_2d(&u.b, CU_TENSOR_MAP_DATA_TYPE_UINT8, w_codes, K / 2, N, K / 2, 128, 128,
                       CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= encode_tmap_2d(&u.la, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, lora, 2 * SVDQ_RANK, M, 2 * SVDQ_RANK * 2, 64, 128,
                       CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= encode_tmap_2d(&u.lb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, lora_up, 2 * SVDQ_RANK, N, 2 * SVDQ_RANK * 2, 64, 128,
                       CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= encode_tmap_2d(&u.y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, y, N, M, (uint64_t)N * 2, 16, 32,
                       CU_TENSOR_MAP_SWIZZLE_32B);
  ok &= encode_tmap_2d(&u.sfa, CU_TENSOR_MAP_DATA_TYPE_UINT8, scales, 256, sfa_rows, 256, 256, 8,
                       CU_TENSOR_MAP_SWIZZLE_NONE);
  ok &= encode_tmap_2d(&u.sfb, CU_TENSOR_MAP_DATA_TYPE_UINT8, w_scales, 256, sfb_rows, 256, 256, 8,
                       CU_TENSOR_MAP_SWIZZLE_NONE);
  ok &= encode_tmap_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, K, M, (uint64_t)K * 2, 64, 128,
                       CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= encode_tmap_2d(&tl, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, lora_down, K, SVDQ_RANK, (uint64_t)K * 2, 64, 32,
                       CU_TENSOR_MAP_SWIZZLE_128B);
  if (!ok) return fail(SVDQ_ERR_CUDA, "cuTensorMapEncodeTiled failed for the fused layer kernel");
  GemmNvfp4Params p{};
  p.M = M;
  p.N = N;
  p.K = K;
  p.act_scales = scales;
  p.w_scales = static_cast<const uint8_t*>(w_scales);
  p.bias = static_cast<const uint16_t*>(bias);
  p.alpha = act_scale * weight_scale;
  p.dev_status = dev_status;
  p.timeout_ns = svdq_timeout_ns();
  // x_hat enters the fp16 down-projection as x_hat * 2^-e (as in the
  // quantize kernel: 2688 s_a maps into [2^12, 2^13)).
  int ex = 0;
  frexpf(2688.0f * act_scale, &ex);
  const int e = ex - 1 - 12;
  FusedQuantParams& q = p.fq;
  q.x = static_cast<const uint16_t*>(x);
  q.inv_smooth = inv_smooth;
  q.l1t = static_cast<const uint16_t*>(lora_down);
  q.act_scale = act_scale;
  q.lr_in_scale = ldexpf(1.0f, -e);
  q.lora_scale = ldexpf(1.0f, e) / (act_scale * weight_scale);
  q.codes = codes;
  q.scales = scales;
  q.lora_act = reinterpret_cast<uint16_t*>(lora);
  q.u_part = reinterpret_cast<float*>(ws + off[4]);
  q.sync = reinterpret_cast<int*>(ws);
  q.splits = fused_splits(K);
  q.row_blocks = (int)(round_up(M, 256) / 128);
  return check_cuda(launch_layer_nvfp4_pair(p, u, tx, tl, stream, pdl), "fused layer kernel launch");
}

int svdq_w4a4_linear(int precision, int M, int N, int K, int rank, const void* x, const float* inv_smooth,
                     const void* lora_down, float act_scale, const void* w_codes, const void* w_scales,
                     float weight_scale, const void* lora_up, const void* bias, void* y, void* workspace,
                     long long workspace_bytes, int* dev_status, void* stream) {
  if (int s = check_gemm_args(precision, M, N, K, rank)) return s;
  if (!workspace) return fail(SVDQ_ERR_INVALID_ARG, "null workspace");
  const long long need = svdq_workspace_bytes(precision, M, N, K, rank);
  if (workspace_bytes < need)
    return fail(SVDQ_ERR_INVALID_ARG, "workspace of %lld bytes is smaller than the %lld needed", workspace_bytes, need);
  if (!aligned16(workspace)) return fail(SVDQ_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
  long long off[6];
  if (int s = svdq_workspace_offsets(precision, M, N, K, rank, off)) return s;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint8_t* codes = ws + off[1];
  uint8_t* scales = ws + off[2];
  uint8_t* lora = ws + off[3];
  // Every argument is checked before the first launch.
  if (!w_codes || !w_scales || !lora_up || !y) return fail(SVDQ_ERR_INVALID_ARG, "null pointer argument");
  if (!aligned16(w_codes) || !aligned16(w_scales) || !aligned16(lora_up) || !aligned16(y) ||
      (bias && !aligned16(bias)))
    return fail(SVDQ_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  int sms = 0;
  if (int s = check_device(&sms)) return s;
  if (int s = resolve_status(&dev_status)) return s;
  if (precision == SVDQ_NVFP4 && use_layer_kernel(M)) {
    if (!x || !inv_smooth || !lora_down) return fail(SVDQ_ERR_INVALID_ARG, "null pointer argument");
    if (!aligned16(x) || !aligned16(inv_smooth) || !aligned16(lora_down))
      return fail(SVDQ_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
    if (!nvfp4_scale_ok(act_scale) || !nvfp4_scale_ok(weight_scale))
      return fail(SVDQ_ERR_INVALID_ARG, "NVFP4 tensor scales must lie in [2^-100, 2^100) (act %g, weight %g)",
                  act_scale, weight_scale);
    return layer_nvfp4_impl(M, N, K, x, inv_smooth, lora_down, act_scale, w_codes, w_scales, weight_scale, lora_up,
                            bias, y, ws, off, dev_status, static_cast<cudaStream_t>(stream), pdl_on());
  }
  const Int4LayerGemm g4 = int4_layer_gemm();
  // INT4 on fp16 operands written out first: when one block per 32 weight
  // rows fits in the SM slots the quantizer leaves free (it runs two 512-
  // thread CTAs per SM, one per 16 rows), extra blocks of the quantizer's
  // launch convert the weight rows beside it; otherwise the operand pass
  // converts both sides after it.  Measured at K = N = 3072: 48.5 against
  // 51.8 us at M = 1024; with too few free slots (M = 4096) the extra blocks
  // lengthen the quantizer's tail instead (115 against 100 us).  The extra
  // blocks stage their rows in the quantizer's 96 KB ring, which bounds K
  // (23552 at most).
  const bool int4_w_side = precision == SVDQ_INT4 && g4 == Int4LayerGemm::kF16Operands &&
                           2 * sms - (int)(round_up(M, 256) / 16) >= (N + 31) / 32 && int4_weight_side_fits(K);
  DequantInt4Params w_side{};
  if (int4_w_side) {
    long long o[7];
    int4_operand_offsets(M, N, K, o);
    w_side = DequantInt4Params{N, K, (int)round_up(N, 256), static_cast<const uint8_t*>(w_codes),
                               static_cast<const uint16_t*>(w_scales), static_cast<const uint16_t*>(lora_up),
                               reinterpret_cast<uint16_t*>(ws + off[4] + o[3]),
                               reinterpret_cast<uint16_t*>(ws + off[4] + o[4]),
                               reinterpret_cast<float*>(ws + off[4] + o[5])};
  }
  if (int s = quantize_act_impl(precision, M, K, rank, x, inv_smooth, lora_down, act_scale, weight_scale, codes,
                                scales, lora, dev_status, stream, int4_w_side ? &w_side : nullptr))
    return s;
  if (precision == SVDQ_INT4) {
    if (g4 == Int4LayerGemm::kI8)
      return gemm_int4_impl(M, N, K, codes, scales, lora, w_codes, w_scales, lora_up, bias, y, dev_status,
                            static_cast<cudaStream_t>(stream), pdl_on(), sms);
    return gemm_int4_f16_impl(M, N, K, codes, scales, lora, w_codes, w_scales, lora_up, bias, y, ws + off[4],
                              dev_status, static_cast<cudaStream_t>(stream), pdl_on(),
                              g4 == Int4LayerGemm::kDequantInGemm, int4_w_side);
  }
  return gemm_nvfp4_impl(M, N, K, codes, scales, lora, w_codes, w_scales, lora_up, bias, act_scale * weight_scale,
                         y, dev_status, static_cast<cudaStream_t>(stream), pdl_on(), sms);
}

// ------------------------------------------------------------------ GELU-MLP fusion

long long svdq_gelu_quant_work_bytes(int M) {
  if (M <= 0) return -1;
  return round_up((int64_t)M * SVDQ_RANK * 4, 256);  // fp32 low-rank sums [M, r]
}

static bool nvfp4_scale_ok(float s) { return s >= 0x1p-100f && s < 0x1p100f; }

// Zero the work buffer and the scale rows no tile of the fused GEMM writes
// (the tiled layout pads rows to 256, the tiles cover a multiple of 128).
static int gelu_quant_prepare(int M, int N, void* next_act_scales, void* work, cudaStream_t stream) {
  if (int s = check_cuda(cudaMemsetAsync(work, 0, svdq_gelu_quant_work_bytes(M), stream), "work memset")) return s;
  const int64_t covered = round_up(M, 128), padded = round_up(M, 256);
  if (padded > covered) {
    const int64_t block = (int64_t)(N / 64) * 512;  // one 128-row block of scales
    uint8_t* base = static_cast<uint8_t*>(next_act_scales) + covered / 128 * block;
    if (int s = check_cuda(cudaMemsetAsync(base, 0, (size_t)block, stream), "scale padding memset")) return s;
  }
  return SVDQ_OK;
}

// h_hat enters the fp16 down-projection as h_hat * 2^-e (the rule of
// svdq_quantize_act: 2688 s maps into [2^12, 2^13)); the finalize step
// multiplies the sums by 2^e / (s s_w).
static int lowrank_exponent(float act_scale) {
  int ex = 0;
  frexpf(2688.0f * act_scale, &ex);
  return ex - 1 - 12;
}

// The fused GEMM, then the conversion of its low-rank sums (PDL-chained).
static int launch_gelu_quant(int M, int N, int K, const void* act_codes, const void* act_scales,
                             const void* lora_act, const void* w_codes, const void* w_scales, const void* lora_up,
                             const void* bias, float alpha, const float* next_inv_smooth, const void* next_lora_down,
                             float next_act_scale, float next_weight_scale, void* next_act_codes,
                             void* next_act_scales, void* next_lora_act, void* work, int* dev_status,
                             cudaStream_t stream, bool pdl, int sms) {
  const int e = lowrank_exponent(next_act_scale);
  GeluQuantParams g{};
  g.inv_smooth = next_inv_smooth;
  g.l1t = static_cast<const uint16_t*>(next_lora_down);
  g.s_d = next_act_scale;
  g.lr_in_scale = ldexpf(1.0f, -e);
  g.codes = static_cast<uint8_t*>(next_act_codes);
  g.scales = static_cast<uint8_t*>(next_act_scales);
  g.u_work = static_cast<float*>(work);
  if (int s = gemm_nvfp4_impl(M, N, K, act_codes, act_scales, lora_act, w_codes, w_scales, lora_up, bias, alpha,
                              nullptr, dev_status, stream, pdl, sms, &g))
    return s;
  const float lora_scale = ldexpf(1.0f, e) / (next_act_scale * next_weight_scale);
  return check_cuda(launch_lowrank_finalize(g.u_work, M, lora_scale, static_cast<uint16_t*>(next_lora_act), stream,
                                            pdl_on()),
                    "low-rank finalize launch");
}

static int check_gelu_quant_args(int M, int N, int K, int rank, float alpha, const float* next_inv_smooth,
                                 const void* next_lora_down, float next_act_scale, float next_weight_scale,
                                 void* next_act_codes, void* next_act_scales, void* next_lora_act, void* work,
                                 long long work_bytes) {
  if (int s = check_gemm_args(SVDQ_NVFP4, M, N, K, rank)) return s;
  if (N % 256 != 0)
    return fail(SVDQ_ERR_UNSUPPORTED_SHAPE, "N=%d must be a multiple of 256 (it is the next layer's K)", N);
  if (!next_inv_smooth || !next_lora_down || !next_act_codes || !next_act_scales || !next_lora_act || !work)
    return fail(SVDQ_ERR_INVALID_ARG, "null pointer argument");
  if (!aligned16(next_inv_smooth) || !aligned16(next_lora_down) || !aligned16(next_act_codes) ||
      !aligned16(next_act_scales) || !aligned16(next_lora_act) || !aligned16(work))
    return fail(SVDQ_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  if (!(alpha > 0.f)) return fail(SVDQ_ERR_INVALID_ARG, "alpha must be positive");
  if (!nvfp4_scale_ok(next_act_scale) || !nvfp4_scale_ok(next_weight_scale))
    return fail(SVDQ_ERR_INVALID_ARG, "NVFP4 tensor scales must lie in [2^-100, 2^100) (act %g, weight %g)",
                next_act_scale, next_weight_scale);
  const long long need = svdq_gelu_quant_work_bytes(M);
  if (work_bytes < need)
    return fail(SVDQ_ERR_INVALID_ARG, "work buffer of %lld bytes is smaller than the %lld needed", work_bytes, need);
  return SVDQ_OK;
}

int svdq_w4a4_gemm_gelu_quant(int M, int N, int K, int rank, const void* act_codes, const void* act_scales,
                              const void* lora_act, const void* w_codes, const void* w_scales, const void* lora_up,
                              const void* bias, float alpha, const float* next_inv_smooth,
                              const void* next_lora_down, float next_act_scale, float next_weight_scale,
                              void* next_act_codes, void* next_act_scales, void* next_lora_act, void* work,
                              long long work_bytes, int* dev_status, void* stream) {
  if (int s = check_gelu_quant_args(M, N, K, rank, alpha, next_inv_smooth, next_lora_down, next_act_scale,
                                    next_weight_scale, next_act_codes, next_act_scales, next_lora_act, work,
                                    work_bytes))
    return s;
  if (!act_codes || !act_scales || !lora_act || !w_codes || !w_scales || !lora_up)
    return fail(SVDQ_ERR_INVALID_ARG, "null pointer argument");
  if (!aligned16(act_codes) || !aligned16(act_scales) || !aligned16(lora_act) || !aligned16(w_codes) ||
      !aligned16(w_scales) || !aligned16(lora_up) || (bias && !aligned16(bias)))
    return fail(SVDQ_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  int sms = 0;
  if (int s = check_device(&sms)) return s;
  if (int s = resolve_status(&dev_status)) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (int s = gelu_quant_prepare(M, N, next_act_scales, work, st)) return s;
  return launch_gelu_quant(M, N, K, act_codes, act_scales, lora_act, w_codes, w_scales, lora_up, bias, alpha,
                           next_inv_smooth, next_lora_down, next_act_scale, next_weight_scale, next_act_codes,
                           next_act_scales, next_lora_act, work, dev_status, st, pdl_on(), sms);
}

long long svdq_mlp_workspace_bytes(int M, int K, int N_hidden, int rank) {
  const long long a = svdq_workspace_bytes(SVDQ_NVFP4, M, N_hidden, K, rank);
  const long long h = svdq_workspace_bytes(SVDQ_NVFP4, M, K, N_hidden, rank);
  const long long w = svdq_gelu_quant_work_bytes(M);
  if (a < 0 || h < 0 || w < 0) return -1;
  return a + h + w;
}

int svdq_w4a4_mlp_gelu(int M, int K, int N_hidden, int rank, const void* x, const float* up_inv_smooth,
                       const void* up_lora_down, float up_act_scale, const void* up_w_codes, const void* up_w_scales,
                       float up_weight_scale, const void* up_lora_up, const void* up_bias,
                       const float* down_inv_smooth, const void* down_lora_down, float down_act_scale,
                       const void* down_w_codes, const void* down_w_scales, float down_weight_scale,
                       const void* down_lora_up, const void* down_bias, void* y, void* workspace,
                       long long workspace_bytes, int* dev_status, void* stream) {
  const int N = N_hidden;
  if (int s = check_gemm_args(SVDQ_NVFP4, M, K, N, rank)) return s;  // the down layer: [M, N] -> [M, K]
  if (!workspace) return fail(SVDQ_ERR_INVALID_ARG, "null workspace");
  const long long need = svdq_mlp_workspace_bytes(M, K, N, rank);
  if (need < 0) return fail(SVDQ_ERR_UNSUPPORTED_SHAPE, "M=%d K=%d N_hidden=%d", M, K, N);
  if (workspace_bytes < need)
    return fail(SVDQ_ERR_INVALID_ARG, "workspace of %lld bytes is smaller than the %lld needed", workspace_bytes, need);
  if (!aligned16(workspace)) return fail(SVDQ_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
  // [the up layer's workspace | the down layer's workspace | the work buffer]
  long long oa[6], oh[6];
  if (int s = svdq_workspace_offsets(SVDQ_NVFP4, M, N, K, rank, oa)) return s;
  if (int s = svdq_workspace_offsets(SVDQ_NVFP4, M, K, N, rank, oh)) return s;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint8_t* a_codes = ws + oa[1];
  uint8_t* a_scales = ws + oa[2];
  uint8_t* a_lora = ws + oa[3];
  uint8_t* hws = ws + oa[5];
  uint8_t* h_codes = hws + oh[1];
  uint8_t* h_scales = hws + oh[2];
  uint8_t* h_lora = hws + oh[3];
  uint8_t* work = hws + oh[5];
  const float up_alpha = up_act_scale * up_weight_scale;
  if (int s = check_gelu_quant_args(M, N, K, rank, up_alpha, down_inv_smooth, down_lora_down, down_act_scale,
                                    down_weight_scale, h_codes, h_scales, h_lora, work,
                                    svdq_gelu_quant_work_bytes(M)))
    return s;
  if (!up_w_codes || !up_w_scales || !up_lora_up || !down_w_codes || !down_w_scales || !down_lora_up || !y)
    return fail(SVDQ_ERR_INVALID_ARG, "null pointer argument");
  if (!aligned16(up_w_codes) || !aligned16(up_w_scales) || !aligned16(up_lora_up) || !aligned16(down_w_codes) ||
      !aligned16(down_w_scales) || !aligned16(down_lora_up) || !aligned16(y) || (up_bias && !aligned16(up_bias)) ||
      (down_bias && !aligned16(down_bias)))
    return fail(SVDQ_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  int sms = 0;
  if (int s = check_device(&sms)) return s;
  if (int s = resolve_status(&dev_status)) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // The memsets go first so that quantize -> fused GEMM -> down GEMM form one
  // chain of programmatic dependent launches.
  if (int s = gelu_quant_prepare(M, N, h_scales, work, st)) return s;
  if (int s = quantize_act_impl(SVDQ_NVFP4, M, K, rank, x, up_inv_smooth, up_lora_down, up_act_scale,
                                up_weight_scale, a_codes, a_scales, a_lora, dev_status, stream))
    return s;
  if (int s = launch_gelu_quant(M, N, K, a_codes, a_scales, a_lora, up_w_codes, up_w_scales, up_lora_up, up_bias,
                                up_alpha, down_inv_smooth, down_lora_down, down_act_scale, down_weight_scale, h_codes,
                                h_scales, h_lora, work, dev_status, st, pdl_on(), sms))
    return s;
  return gemm_nvfp4_impl(M, K, N, h_codes, h_scales, h_lora, down_w_codes, down_w_scales, down_lora_up, down_bias,
                         down_act_scale * down_weight_scale, y, dev_status, st, pdl_on(), sms);
}

// ------------------------------------------------------------------ QKV + RMSNorm + RoPE

static int check_qkv_args(int M, int N, int K, int rank, int heads, int head_dim, const float* gamma_q,
                          const float* gamma_k, const float* rope_cos, const float* rope_sin, void* y) {
  if (head_dim != 128) return fail(SVDQ_ERR_UNSUPPORTED_SHAPE, "head_dim=%d; this build supports 128", head_dim);
  if (heads <= 0 || (long long)N != 3ll * heads * head_dim)
    return fail(SVDQ_ERR_UNSUPPORTED_SHAPE, "N=%d must be 3 * heads * head_dim (heads=%d)", N, heads);
  if (int s = check_gemm_args(SVDQ_NVFP4, M, N, K, rank)) return s;
  if (!gamma_q || !gamma_k || !rope_cos || !rope_sin || !y) return fail(SVDQ_ERR_INVALID_ARG, "null pointer argument");
  if (!aligned16(gamma_q) || !aligned16(gamma_k) || !aligned16(rope_cos) || !aligned16(rope_sin) || !aligned16(y))
    return fail(SVDQ_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  return SVDQ_OK;
}

static QkvParams qkv_params(int heads, const float* gamma_q, const float* gamma_k, const float* rope_cos,
                            const float* rope_sin, void* y) {
  QkvParams q{};
  q.gamma_q = gamma_q;
  q.gamma_k = gamma_k;
  q.rope_cos = rope_cos;
  q.rope_sin = rope_sin;
  q.eps = 1e-6f;
  q.hd = heads * 128;
  q.y = static_cast<uint16_t*>(y);
  return q;
}

int svdq_w4a4_gemm_qkv_norm_rope(int M, int N, int K, int rank, const void* act_codes, const void* act_scales,
                                 const void* lora_act, const void* w_codes, const void* w_scales,
                                 const void* lora_up, const void* bias, float alpha, int heads, int head_dim,
                                 const float* gamma_q, const float* gamma_k, const float* rope_cos,
                                 const float* rope_sin, void* y, int* dev_status, void* stream) {
  if (int s = check_qkv_args(M, N, K, rank, heads, head_dim, gamma_q, gamma_k, rope_cos, rope_sin, y)) return s;
  if (!act_codes || !act_scales || !lora_act || !w_codes || !w_scales || !lora_up)
    return fail(SVDQ_ERR_INVALID_ARG, "null pointer argument");
  if (!aligned16(act_codes) || !aligned16(act_scales) || !aligned16(lora_act) || !aligned16(w_codes) ||
      !aligned16(w_scales) || !aligned16(lora_up) || (bias && !aligned16(bias)))
    return fail(SVDQ_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  if (!(alpha > 0.f)) return fail(SVDQ_ERR_INVALID_ARG, "alpha must be positive");
  int sms = 0;
  if (int s = check_device(&sms)) return s;
  if (int s = resolve_status(&dev_status)) return s;
  const QkvParams q = qkv_params(heads, gamma_q, gamma_k, rope_cos, rope_sin, y);
  return gemm_nvfp4_impl(M, N, K, act_codes, act_scales, lora_act, w_codes, w_scales, lora_up, bias, alpha, y,
                         dev_status, static_cast<cudaStream_t>(stream), pdl_on(), sms, nullptr, &q);
}

int svdq_w4a4_qkv_norm_rope_linear(int M, int K, int heads, int head_dim, int rank, const void* x,
                                   const float* inv_smooth, const void* lora_down, float act_scale,
                                   const void* w_codes, const void* w_scales, float weight_scale,
                                   const void* lora_up, const void* bias, const float* gamma_q, const float* gamma_k,
                                   const float* rope_cos, const float* rope_sin, void* y, void* workspace,
                                   long long workspace_bytes, int* dev_status, void* stream) {
  const int N = 3 * heads * head_dim;
  if (int s = check_qkv_args(M, N, K, rank, heads, head_dim, gamma_q, gamma_k, rope_cos, rope_sin, y)) return s;
  if (!workspace) return fail(SVDQ_ERR_INVALID_ARG, "null workspace");
  const long long need = svdq_workspace_bytes(SVDQ_NVFP4, M, N, K, rank);
  if (workspace_bytes < need)
    return fail(SVDQ_ERR_INVALID_ARG, "workspace of %lld bytes is smaller than the %lld needed", workspace_bytes, need);
  if (!aligned16(workspace)) return fail(SVDQ_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
  if (!w_codes || !w_scales || !lora_up) return fail(SVDQ_ERR_INVALID_ARG, "null pointer argument");
  if (!aligned16(w_codes) || !aligned16(w_scales) || !aligned16(lora_up) || (bias && !aligned16(bias)))
    return fail(SVDQ_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  long long off[6];
  if (int s = svdq_workspace_offsets(SVDQ_NVFP4, M, N, K, rank, off)) return s;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint8_t* codes = ws + off[1];
  uint8_t* scales = ws + off[2];
  uint8_t* lora = ws + off[3];
  int sms = 0;
  if (int s = check_device(&sms)) return s;
  if (int s = resolve_status(&dev_status)) return s;
  if (int s = quantize_act_impl(SVDQ_NVFP4, M, K, rank, x, inv_smooth, lora_down, act_scale, weight_scale, codes,
                                scales, lora, dev_status, stream))
    return s;
  const QkvParams q = qkv_params(heads, gamma_q, gamma_k, rope_cos, rope_sin, y);
  return gemm_nvfp4_impl(M, N, K, codes, scales, lora, w_codes, w_scales, lora_up, bias, act_scale * weight_scale,
                         y, dev_status, static_cast<cudaStream_t>(stream), pdl_on(), sms, nullptr, &q);
}

int awq_w4a16_linear(int M, int N, int K, const void* x, const void* qweight, const void* scales, const void* zeros,
                     const void* bias, void* y, void* stream) {
  if (M <= 0 || N <= 0 || K <= 0) return fail(SVDQ_ERR_UNSUPPORTED_SHAPE, "M=%d N=%d K=%d must be positive", M, N, K);
  if (N % 16 != 0) return fail(SVDQ_ERR_UNSUPPORTED_SHAPE, "N=%d must be a multiple of 16", N);
  if (K % 128 != 0) return fail(SVDQ_ERR_UNSUPPORTED_SHAPE, "K=%d must be a multiple of 128", K);
  if (!x || !qweight || !scales || !zeros || !y) return fail(SVDQ_ERR_INVALID_ARG, "null pointer argument");
  if (!aligned16(x) || !aligned16(qweight) || !aligned16(y) || ((uintptr_t)scales & 1) || ((uintptr_t)bias & 1))
    return fail(SVDQ_ERR_INVALID_ARG, "x, qweight and y must be 16-byte aligned; scales and bias 2-byte aligned");
  int sms = 0;
  if (int s = check_device(&sms)) return s;
  // Token rows are independent: process them 16 at a time (one weight pass each).
  for (int m0 = 0; m0 < M; m0 += 16) {
    AwqParams p{};
    p.M = M - m0 < 16 ? M - m0 : 16;
    p.N = N;
    p.K = K;
    p.x = static_cast<const uint16_t*>(x) + (size_t)m0 * K;
    p.qweight = static_cast<const uint8_t*>(qweight);
    p.scales = static_cast<const uint16_t*>(scales);
    p.zeros = static_cast<const uint8_t*>(zeros);
    p.bias = static_cast<const uint16_t*>(bias);
    p.y = static_cast<uint16_t*>(y) + (size_t)m0 * N;
    if (int s = check_cuda(launch_awq(p, sms, static_cast<cudaStream_t>(stream), pdl_on()), "awq launch")) return s;
  }
  return SVDQ_OK;
}

}  // extern "C"
