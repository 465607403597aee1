/*
 * svdq.h -- C ABI of the B200 (sm_100a) SVDQuant W4A4 / AWQ W4A16 linear layers.
 *
 * The layer (pages: "Hugging Face integrates Nunchaku 4-bit diffusion
 * inference into Diffusers", section "SVDQuant and the Nunchaku engine";
 * "Nunchaku Lite" Diffusers docs, "Supported quantization types" table):
 *
 *   y = (x diag(lambda)^-1) L1 L2 + Q(x diag(lambda)^-1) Q(R)^T + b,
 *   R = W diag(lambda) - (L1 L2)^T,
 *
 * with a 16-bit rank-r branch L1 [K,r], L2 [r,N] (r = 32) and a 4-bit
 * residual: NVFP4 (E2M1 codes, an E4M3 scale per 16 elements, an fp32
 * per-tensor scale) or INT4 (signed, a bf16 scale per 64 elements).
 *
 * Conventions for every call:
 *  - All integers are element counts.  Matrices are row-major; x is [M,K],
 *    W is [N,K] (nn.Linear layout), y is [M,N].  bf16 data is passed as its
 *    16-bit patterns.
 *  - "device" pointers are CUDA device addresses owned by the caller (for
 *    example torch tensors); "host" pointers are ordinary host memory owned by
 *    the caller.  The library never allocates, frees or retains a pointer.
 *  - Device pointers must be 16-byte aligned.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Device calls are asynchronous on that stream; errors found
 *    before launch are returned synchronously, nothing is launched then.
 *  - Return value: an svdq_status.  svdq_last_error() gives a thread-local
 *    message for the last failure.  No C++ exception crosses this boundary.
 *  - `dev_status` is a device int32 the kernels set to a nonzero code when
 *    one of their bounded internal waits gives up; the kernel then drains
 *    its copies, frees its tensor memory and exits, and the outputs of that
 *    call are not valid.  The caller reads it after synchronizing and should
 *    clear it beforehand.  When the caller passes NULL (and for
 *    svdq_quantize_act, which takes no status argument) the kernels report
 *    to the library's own status word on the current device instead, which
 *    svdq_device_status() reads; a timed-out call is never silent.
 *  - Device calls require a compute-capability 10.0 GPU (B200) as the
 *    current device, else SVDQ_ERR_UNSUPPORTED_DEVICE.  There is no fallback.
 *  - Every kernel is launched with programmatic dependent launch: it may be
 *    scheduled while the previous work on the stream finishes, and waits for
 *    that work's completion before it touches global memory.  Setting the
 *    environment variable SVDQ_PDL=0 launches plainly (read at every call).
 *  - Kernel choice (environment, read at every call; results are the same
 *    either way, bit for bit up to the summation order of fp32 low-rank
 *    partials): the NVFP4 GEMMs run on CTA pairs (256 x 256 tiles on two
 *    SMs) for the plain and QKV epilogues and one CTA per 128 x 256 tile for
 *    the GELU-MLP epilogue; SVDQ_NVFP4_GEMM_KERNEL=pair or =single forces
 *    one kind for every call.  NVFP4 activation quantization uses the
 *    TMA-fed kernel; SVDQ_NVFP4_QUANT_KERNEL=copy selects the per-thread-copy
 *    kernel.
 */
#ifndef SVDQ_H
#define SVDQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SVDQ_VERSION 1
#define SVDQ_RANK 32 /* the rank this build supports ("rank": 32 in the docs' config example) */

typedef enum {
  SVDQ_OK = 0,
  SVDQ_ERR_INVALID_ARG = 1,        /* null / misaligned pointer, bad enum, bad scale */
  SVDQ_ERR_UNSUPPORTED_SHAPE = 2,  /* a shape rule below is broken */
  SVDQ_ERR_UNSUPPORTED_DEVICE = 3, /* current device is not sm_100 */
  SVDQ_ERR_CUDA = 4,               /* a CUDA runtime / driver call failed */
  SVDQ_ERR_DEVICE_TIMEOUT = 5      /* reported through dev_status, never returned */
} svdq_status;

/* "precision" of svdq_w4a4 in the "Supported quantization types" table:
 * nvfp4 with group size 16, int4 with group size 64. */
typedef enum { SVDQ_NVFP4 = 0, SVDQ_INT4 = 1 } svdq_precision;

const char* svdq_status_string(int status);
const char* svdq_last_error(void);
int svdq_version(void);

/* Upper bound, in nanoseconds, on any single internal wait of a GEMM kernel
 * before it gives up and reports through dev_status (default 1e9).  Affects
 * launches made after the call, from any thread. */
void svdq_set_timeout_ns(unsigned long long ns);
unsigned long long svdq_get_timeout_ns(void);

/* svdq_device_status: the library's own status word on the current device
 * (the one kernels report to when their caller passed dev_status == NULL).
 * Waits for `stream` to finish, stores the word in *value (host int; 0 when
 * no wait has given up since the word was last cleared) and, if `clear` is
 * nonzero, resets it to 0.  The word lives in a file-scope device variable of
 * this library, one per device context; calls that race with kernels
 * reporting to it on other streams see either value. */
int svdq_device_status(int* value, int clear, void* stream);

/* ------------------------------------------------------------------ layouts
 * Codes: 4-bit values, two per byte, element 2j in the low nibble of byte j
 * of its row.  NVFP4 codes are E2M1 (bit 3 = sign); INT4 codes are two's
 * complement in [-7, 7].
 *
 * NVFP4 scales ("tiled" layout, what the block-scaled MMA consumes): E4M3
 * bytes, rows padded with zeros to a multiple of 256.  Scale (row m, group g),
 * g = k/16, sits at byte
 *     ((m/128) * (K/64) + g/4) * 512 + (m%32) * 16 + ((m%128)/32) * 4 + g%4.
 * INT4 scales: bf16, group-major [K/64][rows padded to 256], zero padded.
 * Sizes in bytes (or -1 for an unsupported precision / K): */
long long svdq_act_scale_bytes(int precision, int M, int K);
long long svdq_weight_scale_bytes(int precision, int N, int K);

/* Host helpers: NVFP4 scales between row-major [rows, K/16] and tiled. */
int svdq_scales_to_rowmajor(int rows, int K, const uint8_t* tiled, uint8_t* rowmajor);
int svdq_scales_from_rowmajor(int rows, int K, const uint8_t* rowmajor, uint8_t* tiled);

/* ------------------------------------------------------------------ host pack
 * svdq_pack_weights: offline weight preparation (host, untimed).
 * "SVDQuant and the Nunchaku engine": outliers migrate into the weights, a
 * 16-bit low-rank branch absorbs the hardest part, the residual is quantized
 * to 4 bits.  Computes, in this order:
 *   inv_smooth[k] = fp32(1 / smooth[k]);
 *   R[n,k] = fp32( W[n,k]*smooth[k] - sum_{t ascending} L1[k,t]*L2[t,n] )
 *            (products and sum in fp64, one rounding to fp32);
 *   NVFP4: s_w = amax|R| / 2688 (1 if R == 0); per 16 along k:
 *          a = max|v|, sb = E4M3_rn_sat(a * fp32(1/fp32(6 s_w))), d = float(sb)*s_w,
 *          code = E2M1_rn_sat(v * fp32(1/d)) (sign kept), all codes 0 when d == 0.
 *   INT4:  per 64 along k: sc = bf16(a / 7), q = clamp(rint(v * fp32(1/sc)), -8, 7).
 * Inputs (host): W bf16 [N,K]; smooth fp32 [K] (lambda, > 0); L1 bf16 [K,r];
 * L2 bf16 [r,N].  Outputs (host, caller-allocated):
 *   codes      [N, K/2] bytes
 *   scales     svdq_weight_scale_bytes(precision, N, K) bytes
 *   weight_scale  1 float (s_w; 1.0 for INT4)
 *   inv_smooth fp32 [K]
 *   lora_down  [r, K] 16-bit (L1 transposed, the down-projection operand):
 *              fp16 for NVFP4 (|L1| must not exceed 65504, else
 *              SVDQ_ERR_INVALID_ARG), bf16 for INT4
 *   lora_up    bf16 [N, 2r]  (row n = [L2[:,n], L2[:,n]], the up-projection
 *                             operand for the hi/lo split activation)
 * Shapes: N % 128 == 0, K % 256 == 0, rank == SVDQ_RANK. */
int svdq_pack_weights(int precision, int N, int K, int rank, const uint16_t* W, const float* smooth,
                      const uint16_t* L1, const uint16_t* L2, uint8_t* codes, uint8_t* scales, float* weight_scale,
                      float* inv_smooth, uint16_t* lora_down, uint16_t* lora_up);

/* ------------------------------------------------------------------ host calibration
 * svdq_calibrate: the offline step that produces a layer's smoothing
 * factors, low-rank factors and static activation scale from its weights
 * and a calibration batch ("SVDQuant and the Nunchaku engine": outliers
 * migrate into the weights; a 16-bit low-rank branch from a decomposition
 * of the weights absorbs their hardest part).  Host only, untimed:
 *   smooth[k] = sqrt(max_i |x[i,k]| / max_n |W[n,k]|) in fp32, 1 where a max is 0;
 *   A = (W diag(smooth))^T [K, N] in fp64;
 *   randomized subspace iteration (Halko, Martinsson & Tropp 2011, Alg. 4.4)
 *   with the caller's Gaussian test matrix omega [N, rank + oversample]
 *   (fp64, row-major) and power_iters iterations: Q = qr(A omega); repeat:
 *   Z = qr(A^T Q), Q = qr(A Z); B = Q^T A = Ub S Vt; U = Q Ub; each column of
 *   U negated if its largest-magnitude entry (the first on a tie) is
 *   negative, with the matching row of Vt;
 *   L1 = bf16(U[:, :rank] S[:rank]) [K, rank], L2 = bf16(Vt[:rank]) [rank, N];
 *   act_scale = max |x[i,k] * fp32(1/smooth[k])| / 2688 (fp32; 1 if 0).
 * Inputs (host): W bf16 [N, K], x bf16 [M, K] (the calibration batch),
 * omega.  Outputs (host, caller-allocated): smooth fp32 [K], L1 and L2 bf16,
 * act_scale (1 float).  The result does not depend on the number of host
 * threads used.  rank + oversample <= min(K, N). */
int svdq_calibrate(int N, int K, int M, int rank, int oversample, int power_iters, const uint16_t* W,
                   const uint16_t* x, const double* omega, float* smooth, uint16_t* L1, uint16_t* L2,
                   float* act_scale);

/* ------------------------------------------------------------------ device
 * svdq_quantize_act: smoothing + activation quantization + low-rank
 * down-projection in one pass over x (the Nunchaku engine's fused
 * "down-projection + quantize" kernel, "SVDQuant and the Nunchaku engine").
 *   x_hat = fp32(x) * inv_smooth;  codes/scales as in svdq_pack_weights with
 *   s = act_scale for NVFP4;  u = x_hat L1;
 *   lora_act[m] = [hi(u*c), lo(u*c)] (bf16 pair whose sum is u*c to ~2^-16),
 *   c = 1/(act_scale*weight_scale) for NVFP4 and 1 for INT4.
 * NVFP4 runs the down-projection on fp16 operands: x_hat * 2^-e with 2^e the
 * power of two mapping 2688*act_scale into [2^12, 2^13), times the fp16
 * lora_down; INT4 uses a bf16 hi+lo split of x_hat.  Both accumulate in fp32.
 * Device inputs: x bf16 [M,K]; inv_smooth fp32 [K]; lora_down [r,K] as packed.
 * Device outputs: act_codes [M, K/2]; act_scales svdq_act_scale_bytes;
 * lora_act bf16 [M, 2r].  act_scale (NVFP4 s_a, e.g. amax|x_hat|/2688) and
 * weight_scale must lie in [2^-100, 2^100) for NVFP4 (so that every block
 * reciprocal is finite) and are ignored for INT4.
 * Shapes: M >= 1, K % 256 == 0, rank == SVDQ_RANK. */
int svdq_quantize_act(int precision, int M, int K, int rank, const void* x, const float* inv_smooth,
                      const void* lora_down, float act_scale, float weight_scale, void* act_codes, void* act_scales,
                      void* lora_act, void* stream);

/* svdq_w4a4_gemm: the 4-bit GEMM with the low-rank up-projection and bias in
 * its epilogue (the engine's fused "up-projection + 4-bit GEMM" kernel), on
 * already-quantized activations:
 *   NVFP4: y = bf16( alpha * ( sum_k deq(a) deq(w) + lora_act . lora_up^T ) + bias )
 *          with alpha = s_a * s_w;
 *   INT4:  y = bf16( sum_g sa[m,g] sw[n,g] sum_{k in g} qa qw + lora_act . lora_up^T + bias ),
 *          the 64-group sums exact in int32 (alpha is ignored).
 * Device inputs as produced by svdq_quantize_act and svdq_pack_weights; bias
 * bf16 [N] or NULL; output y bf16 [M,N].
 * Shapes: M >= 1, N % 128 == 0, K % 256 == 0. */
int svdq_w4a4_gemm(int precision, int M, int N, int K, int rank, const void* act_codes, const void* act_scales,
                   const void* lora_act, const void* w_codes, const void* w_scales, const void* lora_up,
                   const void* bias, float alpha, void* y, int* dev_status, void* stream);

/* svdq_w4a4_linear: the whole layer, y = svdq_w4a4_gemm(svdq_quantize_act(x))
 * on `stream`: svdq_quantize_act then svdq_w4a4_gemm, the GEMM launched with
 * programmatic dependent launch so that its prologue overlaps the quantize
 * kernel's tail.
 *  - INT4: the product runs on the fp16 tensor pipe instead of svdq_w4a4_gemm's
 *    i8 kernel (which has no scratch): both operands are first written out
 *    to the workspace as fp16 values, exactly sa*qa and sw*qw (an 8-bit
 *    scale significand times a code of at most 3 bits fits fp16's 11), each
 *    row scaled by a power of two 2^-E (E = floor(log2 of the row's largest
 *    scale) - 12, clamped to [-100, 100]) that the epilogue undoes; exact for
 *    every group within 2^29 of its row's largest scale while that scale
 *    lies in [2^-88, 2^113) (E not clamped).  A row whose largest scale is
 *    2^113 or more (values near 10^34) overflows the fp16 operand: use
 *    SVDQ_INT4_LAYER_GEMM=i8 for such data.  Same products,
 *    summed in fp32 in another order, so y can differ from quantize + gemm in
 *    its last bits.  SVDQ_INT4_LAYER_GEMM in the environment (read at every
 *    call) selects "dq" (the GEMM builds the fp16 tiles itself in shared
 *    memory; the same y bit for bit, slower) or "i8" (svdq_w4a4_gemm's
 *    kernel).
 *  - With SVDQ_LAYER_KERNEL=fused in the environment (read at every call;
 *    NVFP4 on the CTA-pair GEMM only): ONE kernel, whose epilogue warps
 *    quantize x themselves, 128 rows x K/splits columns at a time (splits =
 *    the largest divisor of K/256 up to 12), while their accumulator is not
 *    ready; each CTA's TMA producer waits (bounded, like every wait of the
 *    library) for its 128 rows to be complete.  Codes and scales are those
 *    of svdq_quantize_act bit for bit; the low-rank activation sums the same
 *    products in a different (fixed) order, so y can differ from quantize +
 *    gemm in its last bits, and is the same on every run.  It is slower than
 *    the two kernels on B200 (the quantizer's arithmetic competes with the
 *    GEMM's MMA issue) and kept for comparison.
 * `workspace` is a device buffer of at least svdq_workspace_bytes(precision,
 * M, N, K, rank) bytes laid out as svdq_workspace_offsets gives:
 *   [0]  control words of the one-kernel layer, a fixed 64 KiB at offset 0;
 *        when that layer runs they MUST BE ZERO before the first call on a
 *        workspace (e.g. a workspace from cudaMemset or torch.zeros), and
 *        every call leaves them zero again (the kernel's last CTA resets
 *        them), so a workspace can be reused by calls of any shape without
 *        clearing it; the two-kernel path does not touch them;
 *   [1]  act codes [M, K/2];  [2] act scales;  [3] lora_act bf16 [M, 2r];
 *   [4]  NVFP4: the one-kernel layer's fp32 low-rank partial sums; INT4: the
 *        fp16 operands of the product (A' [M, K], the scaled lora_act
 *        [M, 2r], the rows' powers of two [M], then W' [N, K], the scaled
 *        lora_up [N, 2r] and [N], each 256-byte aligned; A' and W' are
 *        not written with SVDQ_INT4_LAYER_GEMM=dq);
 *   [5]  the end (= the size).
 * N (the layer's output width) sizes only the INT4 region; NVFP4 accepts any
 * N >= 0.
 * Calls that share a workspace must not overlap in time.  The one-kernel
 * layer takes M up to 1040384 (larger M runs as two kernels). */
long long svdq_workspace_bytes(int precision, int M, int N, int K, int rank);
int svdq_workspace_offsets(int precision, int M, int N, int K, int rank, long long* offsets /* [6], host */);
int svdq_w4a4_linear(int precision, int M, int N, int K, int rank, const void* x, const float* inv_smooth,
                     const void* lora_down, float act_scale, const void* w_codes, const void* w_scales,
                     float weight_scale, const void* lora_up, const void* bias, void* y, void* workspace,
                     long long workspace_bytes, int* dev_status, void* stream);

/* ------------------------------------------------------------------ no-allocation variant
 * svdq_w4a4_linear_noalloc: the same layer as svdq_w4a4_linear, for callers
 * that cannot allocate device memory when they run it -- code recorded into a
 * CUDA graph on a stream someone else captures, plugins that receive only
 * input and output pointers from a host framework that owns all memory, or
 * allocators that forbid allocations after start-up.  The pages have no
 * counterpart to this entry point; it is a deployment convenience.
 * Instead of a caller workspace it uses a file-scope device array of
 * SVDQ_NOALLOC_SCRATCH_BYTES (32 MiB) that the CUDA driver reserves on every
 * GPU that loads the library, until the process exits.  It never calls
 * cudaMalloc, cudaFree or any allocating routine.
 *  - Limit: svdq_workspace_bytes(precision, M, N, K, rank) must not exceed
 *    SVDQ_NOALLOC_SCRATCH_BYTES (e.g. M = 4096 tokens up to K = 9216, or
 *    2048 tokens up to K = 12288, for NVFP4); larger shapes return
 *    SVDQ_ERR_UNSUPPORTED_SHAPE with a message.
 *  - The first call on a device looks up the array's device address with
 *    cudaGetSymbolAddress (once per device and driver context, with that
 *    device current; after a cudaDeviceReset the next call looks it up
 *    again); make that first call before any stream capture.
 *  - All calls share the one array, which keeps the last call's contents.
 *    Its first 64 KiB are the layer kernel's control words (see
 *    svdq_w4a4_linear): the array is zero when the module loads and every
 *    call leaves those words zero again.  Calls whose kernels overlap on the
 *    GPU (different streams without ordering, or concurrent threads) race on
 *    it: order them on one stream.
 * Arguments, layouts and errors are those of svdq_w4a4_linear without the
 * workspace pair. */
#define SVDQ_NOALLOC_SCRATCH_BYTES (32ll << 20)
long long svdq_noalloc_scratch_bytes(void);
int svdq_w4a4_linear_noalloc(int precision, int M, int N, int K, int rank, const void* x, const float* inv_smooth,
                             const void* lora_down, float act_scale, const void* w_codes, const void* w_scales,
                             float weight_scale, const void* lora_up, const void* bias, void* y, int* dev_status,
                             void* stream);

/* ------------------------------------------------------------------ GELU-MLP fusion
 * "Nunchaku Lite" docs, section "Fused kernels": the original engine runs a
 * diffusion transformer's MLP (up projection, GELU, down projection) with a
 * fused GELU kernel.
 *
 * svdq_w4a4_gemm_gelu_quant: the up layer's NVFP4 GEMM (svdq_w4a4_gemm's
 * arguments up to alpha) whose output
 *   v = alpha * ( sum_k deq(a) deq(w) + lora_act . lora_up^T ) + bias      (fp32)
 * is never stored: it goes through h = GELU(v) = v Phi(v) (the exact erf
 * form), the NEXT layer's smoothing h_hat = h * next_inv_smooth[n] and the
 * next layer's activation side exactly as svdq_quantize_act defines it for
 * NVFP4 with s_a = next_act_scale: E2M1 codes with an E4M3 scale per 16
 * (written to next_act_codes [M, N/2] and next_act_scales,
 * svdq_act_scale_bytes(SVDQ_NVFP4, M, N) bytes, padding rows zero) and the
 * low-rank activation next_lora_act bf16 [M, 2r] = [hi | lo] of
 * (h_hat L1_next) / (next_act_scale * next_weight_scale), computed on fp16
 * operands (h_hat * 2^-e with 2^e as in svdq_quantize_act, and
 * next_lora_down [r, N] as packed) with fp32 accumulation.  The sum over N of
 * the low-rank partials uses fp32 atomic adds, so next_lora_act can differ
 * between runs in its last bits; codes and scales are deterministic.
 * `work` is device scratch of svdq_gelu_quant_work_bytes(M) bytes (the fp32
 * low-rank sums) that the call zeroes on `stream` before use; calls sharing
 * it must not overlap.  The call launches a memset, the GEMM and a small
 * kernel that converts the sums to next_lora_act.
 * The outputs feed svdq_w4a4_gemm of the next layer directly.
 * Shapes: M >= 1, N % 256 == 0 (N is the next layer's K), K % 256 == 0,
 * rank == SVDQ_RANK.  NVFP4 only; scales in [2^-100, 2^100). */
long long svdq_gelu_quant_work_bytes(int M);
int svdq_w4a4_gemm_gelu_quant(int M, int N, int K, int rank, const void* act_codes, const void* act_scales,
                              const void* lora_act, const void* w_codes, const void* w_scales, const void* lora_up,
                              const void* bias, float alpha, const float* next_inv_smooth,
                              const void* next_lora_down, float next_act_scale, float next_weight_scale,
                              void* next_act_codes, void* next_act_scales, void* next_lora_act, void* work,
                              long long work_bytes, int* dev_status, void* stream);

/* svdq_w4a4_mlp_gelu: the MLP block y = down(GELU(up(x))) with two NVFP4
 * svdq_w4a4 layers, up: [M, K] -> [M, N_hidden], down: [M, N_hidden] ->
 * [M, K]: svdq_quantize_act of x for the up layer, then
 * svdq_w4a4_gemm_gelu_quant, then the down layer's svdq_w4a4_gemm, all on
 * `stream` (the GEMMs with programmatic dependent launch).  Each layer's
 * arguments are those of svdq_w4a4_linear (inv_smooth, lora_down, act_scale,
 * w_codes, w_scales, weight_scale, lora_up, bias as packed).  x and y are
 * bf16 [M, K]; `workspace` is device memory of at least
 * svdq_mlp_workspace_bytes(M, K, N_hidden, rank) bytes holding both layers'
 * quantized activations and the fused GEMM's work buffer; calls sharing it
 * must not overlap.  Shapes: K % 256 == 0, N_hidden % 256 == 0. */
long long svdq_mlp_workspace_bytes(int M, int K, int N_hidden, int rank);
int svdq_w4a4_mlp_gelu(int M, int K, int N_hidden, int rank, const void* x, const float* up_inv_smooth,
                       const void* up_lora_down, float up_act_scale, const void* up_w_codes, const void* up_w_scales,
                       float up_weight_scale, const void* up_lora_up, const void* up_bias,
                       const float* down_inv_smooth, const void* down_lora_down, float down_act_scale,
                       const void* down_w_codes, const void* down_w_scales, float down_weight_scale,
                       const void* down_lora_up, const void* down_bias, void* y, void* workspace,
                       long long workspace_bytes, int* dev_status, void* stream);

/* ------------------------------------------------------------------ QKV + RMSNorm + RoPE
 * "Nunchaku Lite" docs, section "Fused kernels": the original engine combines
 * the Q, K and V projections with RMSNorm and RoPE.
 *
 * svdq_w4a4_gemm_qkv_norm_rope: the fused QKV projection's NVFP4 GEMM
 * (svdq_w4a4_gemm's arguments up to alpha) whose output
 *   v = alpha * ( sum_k deq(a) deq(w) + lora_act . lora_up^T ) + bias   (fp32)
 * is, per row and before rounding, treated as [Q | K | V] with `heads` heads
 * of head_dim = 128 features each (head h of a part in its columns
 * [128 h, 128 h + 128)):
 *   Q and K heads: u = v / sqrt(mean(v^2) + 1e-6) * gamma (gamma_q for Q,
 *                  gamma_k for K, fp32 [128]), then each feature pair
 *                  (u[2i], u[2i+1]) is rotated by the row's angle i:
 *                  (a, b) -> (a cos - b sin, a sin + b cos) with
 *                  cos = rope_cos[i * M + m], sin = rope_sin[i * M + m]
 *                  (fp32 [64, M], pair-major: the tables of all tokens for
 *                  pair 0, then pair 1, ...);
 *   V heads:       unchanged;
 * then rounded to bf16 into y [M, N].  N = 3 * heads * 128, K % 256 == 0.
 *
 * svdq_w4a4_qkv_norm_rope_linear: svdq_quantize_act of x then the call above,
 * with svdq_w4a4_linear's arguments and workspace; the weights must be those
 * of a [3 * heads * head_dim, K] layer (N is derived from heads, so the
 * library cannot check it against the buffers). */
int svdq_w4a4_gemm_qkv_norm_rope(int M, int N, int K, int rank, const void* act_codes, const void* act_scales,
                                 const void* lora_act, const void* w_codes, const void* w_scales,
                                 const void* lora_up, const void* bias, float alpha, int heads, int head_dim,
                                 const float* gamma_q, const float* gamma_k, const float* rope_cos,
                                 const float* rope_sin, void* y, int* dev_status, void* stream);
int svdq_w4a4_qkv_norm_rope_linear(int M, int K, int heads, int head_dim, int rank, const void* x,
                                   const float* inv_smooth, const void* lora_down, float act_scale,
                                   const void* w_codes, const void* w_scales, float weight_scale,
                                   const void* lora_up, const void* bias, const float* gamma_q, const float* gamma_k,
                                   const float* rope_cos, const float* rope_sin, void* y, void* workspace,
                                   long long workspace_bytes, int* dev_status, void* stream);

/* ------------------------------------------------------------------ AWQ W4A16
 * "Nunchaku Lite" docs, "Supported quantization types" table: awq_w4a16,
 * int4, group size 64 -- an INT4 weight-only AWQ-style kernel for the
 * memory-bound modulation (adaptive-norm) projections.  Asymmetric uint4 with
 * an integer zero point per 64 along K:
 *   mx, mn = max, min of the group; rng = mx - mn (|mx| if 0, then 1 if 0);
 *   sc = bf16(rng / 15); z = clamp(rint(-mn / sc), 0, 15);
 *   q = clamp(rint(w / sc) + z, 0, 15);  deq = (q - z) * sc.
 * awq_pack_weights (host): W bf16 [N,K] -> qweight [N, K/2] (two codes per
 * byte, element 2j low nibble), scales bf16 [N, K/64], zeros [N, K/128]
 * (group 2j in the low nibble).  K % 128 == 0.
 * awq_w4a16_linear (device): y bf16 [M,N] = bf16(x deq^T + bias), x bf16
 * [M,K], bias bf16 [N] or NULL.  Rows are processed 16 at a time (each group
 * of 16 rows streams the weight once).  N % 16 == 0, K % 128 == 0. */
int awq_pack_weights(int N, int K, const uint16_t* W, uint8_t* qweight, uint16_t* scales, uint8_t* zeros);
int awq_w4a16_linear(int M, int N, int K, const void* x, const void* qweight, const void* scales, const void* zeros,
                     const void* bias, void* y, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* SVDQ_H */
