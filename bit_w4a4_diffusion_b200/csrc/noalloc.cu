// svdq_w4a4_linear_noalloc: the whole W4A4 layer without a caller-provided
// workspace and without allocating any device memory.
//
// Some callers cannot call cudaMalloc at the point where they run the layer:
// code running while a CUDA graph is being captured on a stream the caller
// does not control, plugins handed only input and output pointers by a host
// framework that owns every allocation, or allocators that forbid extra
// device allocations after start-up.  For them the quantized activations that
// svdq_w4a4_linear keeps in its workspace live instead in a file-scope device
// array of SVDQ_NOALLOC_SCRATCH_BYTES that the CUDA driver sets aside when it
// loads this module; every GPU that loads the library holds it until the
// process exits.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "svdq.h"
#include "svdq_internal.h"

namespace {

static __device__ __align__(256) uint8_t g_noalloc_scratch[SVDQ_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
struct ScratchSlot {
  unsigned long long ctx_id = 0;   // context the address belongs to
  void* ptr = nullptr;
};
ScratchSlot g_scratch[kMaxDevices];
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device.  In host code
// the array's name is only a host-side stand-in, so the address must come
// from cudaGetSymbolAddress, with that device current.  It is looked up once
// per device and context: a device reset (or another driver context) loads
// the module again, possibly at another address, so the cached address is
// dropped whenever the current context's id differs from the one it was
// taken in.
int scratch_for_current_device(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return svdq::record_error(SVDQ_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices)
    return svdq::record_error(SVDQ_ERR_UNSUPPORTED_DEVICE, "device index %d out of range", dev);
  const unsigned long long ctx = svdq::current_context_id();
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  ScratchSlot& slot = g_scratch[dev];
  if (slot.ptr == nullptr || ctx == 0 || slot.ctx_id != ctx) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr)
      return svdq::record_error(SVDQ_ERR_CUDA, "cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
    slot.ptr = p;
    slot.ctx_id = ctx;
  }
  *out = slot.ptr;
  return SVDQ_OK;
}

}  // namespace

extern "C" {

long long svdq_noalloc_scratch_bytes(void) { return (long long)SVDQ_NOALLOC_SCRATCH_BYTES; }

int svdq_w4a4_linear_noalloc(int precision, int M, int N, int K, int rank, const void* x, const float* inv_smooth,
                             const void* lora_down, float act_scale, const void* w_codes, const void* w_scales,
                             float weight_scale, const void* lora_up, const void* bias, void* y, int* dev_status,
                             void* stream) {
  const long long need = svdq_workspace_bytes(precision, M, N, K, rank);
  if (need < 0) {
    // Let the regular entry point produce its precise shape / argument error.
    return svdq_w4a4_linear(precision, M, N, K, rank, x, inv_smooth, lora_down, act_scale, w_codes, w_scales,
                            weight_scale, lora_up, bias, y, nullptr, 0, dev_status, stream);
  }
  if (need > (long long)SVDQ_NOALLOC_SCRATCH_BYTES)
    return svdq::record_error(SVDQ_ERR_UNSUPPORTED_SHAPE,
                              "M=%d N=%d K=%d needs %lld bytes of scratch; the built-in scratch holds %lld bytes "
                              "(use svdq_w4a4_linear with a workspace)",
                              M, N, K, need, (long long)SVDQ_NOALLOC_SCRATCH_BYTES);
  void* scratch = nullptr;
  if (int s = scratch_for_current_device(&scratch)) return s;
  // The scratch's first 64 KiB are the layer kernel's control words: zero
  // when the module is loaded (a file-scope device array starts zeroed) and
  // left zero by every call.  The rest needs no clearing: the layer writes
  // every byte it uses (code rows < M, scale rows up to the 256-row padding,
  // low-rank rows < M, the partial sums, and for INT4 the fp16 operand rows
  // < M and < N with their powers of two) before reading it.
  return svdq_w4a4_linear(precision, M, N, K, rank, x, inv_smooth, lora_down, act_scale, w_codes, w_scales,
                          weight_scale, lora_up, bias, y, scratch, need, dev_status, stream);
}

}  // extern "C"
