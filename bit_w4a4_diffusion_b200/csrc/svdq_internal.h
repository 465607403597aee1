// Internal launch interfaces shared by the C-ABI layer and the kernels.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace svdq {

// Every kernel of the library waits for its stream predecessor with
// griddepcontrol.wait before it touches global memory, so any launch may
// carry the programmatic-dependent-launch attribute: the kernel's prologue
// then overlaps the predecessor's tail.
inline void set_pdl(cudaLaunchConfig_t& cfg, cudaLaunchAttribute (&attr)[1], bool pdl) {
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
}

// Device-status codes written by bounded waits (0 = fine).
enum DeviceStatus : int {
  kDevOk = 0,
  kDevTimeoutProducer = 1,
  kDevTimeoutMma = 2,
  kDevTimeoutEpilogue = 3,
  kDevTimeoutDrain = 4,
};

// INT4 rows -> exact fp16 operands for the fp16 tensor pipe (dequant_int4.cu):
// out[r, k] = fp16(s[r, k/64] 2^-E[r] q[r, k]) with K permuted within every
// 8-code word as (0, 2, 4, 6, 1, 3, 5, 7), lora_out = lora_in 2^-E[r],
// factor[r] = 2^E[r].
struct DequantInt4Params {
  int R, K, R_pad;
  const uint8_t* codes;       // [R, K/2]
  const uint16_t* scales;     // bf16 [K/64][R_pad]
  const uint16_t* lora_in;    // bf16 [R, 64] or null
  uint16_t* out;              // fp16 [R, K], or null: only factor and lora_out
  uint16_t* lora_out;         // bf16 [R, 64] (unused when lora_in is null)
  float* factor;              // fp32 [R]
};

struct QuantActParams {
  int M, K, M_pad;            // M_pad: rows of the scale buffer (multiple of 256)
  const uint16_t* x;          // bf16 [M, K]
  const float* inv_smooth;    // fp32 [K]
  const uint16_t* lora_down;  // [r, K] (L1 transposed): fp16 for NVFP4, bf16 for INT4
  float act_scale;            // NVFP4 per-tensor activation scale s_a
  float lora_scale;           // multiplier folded into lora_act: 2^e/(s_a s_w) (NVFP4) or 1
  float lr_in_scale;          // NVFP4: 2^-e applied to x_hat before its fp16 conversion
  uint8_t* act_codes;         // [M, K/2]
  uint8_t* act_scales;        // NVFP4: tiled e4m3; INT4: bf16 [K/64][M_pad]
  uint16_t* lora_act;         // bf16 [M, 2r]  (hi | lo)
  // INT4: blocks s1_blocks .. s1_blocks + w_blocks - 1 of the launch convert
  // the rows of w_side (the layer's weight operand, int4_dequant_rows.cuh)
  // beside the quantizer, 32 rows at a time; w_side.R = 0: none.
  DequantInt4Params w_side;
  int s1_blocks;
  int w_blocks;
};

cudaError_t launch_quantize_act(const QuantActParams& p, bool nvfp4, cudaStream_t stream, bool pdl);
// Whether the INT4 quantizer's shared-memory ring holds the staging of its
// weight-side blocks (32 rows of length K) as well.
bool int4_weight_side_fits(int K);
// NVFP4, TMA-fed: x [M, K] bf16 and L1^T [32, K] fp16 as 64 x 32 SWIZZLE_128B boxes.
cudaError_t launch_quantize_nvfp4(const QuantActParams& p, const CUtensorMap& tm_x, const CUtensorMap& tm_l1t,
                                  int* dev_status, unsigned long long timeout_ns, cudaStream_t stream, bool pdl);

// The GELU-MLP epilogue: the up layer's output never leaves the chip; the
// epilogue applies GELU and the down layer's smoothing, quantizer and
// low-rank down-projection (partial sums over N tiles added into u_work,
// converted to lora_act by launch_lowrank_finalize afterwards).
struct GeluQuantParams {
  const float* inv_smooth;    // down layer 1/lambda, fp32 [N]
  const uint16_t* l1t;        // down layer lora_down, fp16 [32, N]
  float s_d;                  // down layer activation tensor scale
  float lr_in_scale;          // 2^-e applied before the fp16 conversion
  uint8_t* codes;             // [M, N/2]
  uint8_t* scales;            // tiled e4m3 with K = N, rows padded to 256
  float* u_work;              // fp32 [M, 32], zero at launch
};

// The QKV epilogue: columns [Q | K | V] of 128-feature heads; RMSNorm with
// per-feature weights over each Q and K head, then rotation of the feature
// pairs (2i, 2i + 1) by the token's angle; V gets only the bias.
struct QkvParams {
  const float* gamma_q;   // fp32 [128]
  const float* gamma_k;   // fp32 [128]
  const float* rope_cos;  // fp32 [64, M] (pair-major)
  const float* rope_sin;  // fp32 [64, M]
  float eps;
  int hd;                 // columns per part: heads * 128
  uint16_t* y;            // bf16 [M, N]
};

// The whole NVFP4 layer in one kernel (svdq_w4a4_linear on CTA pairs): the
// GEMM's epilogue warps quantize x themselves, one unit of 128 rows x K/splits
// columns at a time, taken in order from a global queue while their
// accumulator is not ready; each CTA's producer waits for its 128-row block
// to be complete before it loads that block's codes, scales and low-rank
// activation.  The low-rank partial sums of a unit go to their own slot of
// u_part; the last unit of a row block adds the slots in slot order (so the
// result does not depend on which CTA ran which unit), writes lora_act and
// raises the block's ready word.
struct FusedQuantParams {
  const uint16_t* x;          // bf16 [M, K]
  const float* inv_smooth;    // fp32 [K]
  const uint16_t* l1t;        // fp16 [32, K] (lora_down)
  float act_scale;            // s_a
  float lora_scale;           // 2^e / (s_a s_w): folded into lora_act
  float lr_in_scale;          // 2^-e applied before the fp16 conversion
  uint8_t* codes;             // [M, K/2]
  uint8_t* scales;            // tiled e4m3, rows padded to 256
  uint16_t* lora_act;         // bf16 [M, 64] = [hi | lo]
  float* u_part;              // fp32 [splits][row_blocks * 128][32]
  int* sync;                  // control words (layout below): zero at launch, left zero
  int splits;                 // units per 128-row block (each K / splits columns)
  int row_blocks;             // rows padded to 256, / 128
};

// Control words of the fused layer kernel, int32 offsets into
// FusedQuantParams::sync (a 64 KiB region): the unit queue, the count of
// CTAs that finished, per row block the count of finished units and the
// ready word, each group on its own cache lines.
constexpr int kSyncQueue = 0;
constexpr int kSyncExit = 32;
constexpr int kSyncCount = 64;
constexpr int kSyncMaxRowBlocks = 8128;
constexpr int kSyncReady = kSyncCount + kSyncMaxRowBlocks;
constexpr long long kSyncBytes = 65536;
static_assert((kSyncReady + kSyncMaxRowBlocks) * 4 <= kSyncBytes, "control words fit the region");

struct GemmNvfp4Params {
  int M, N, K;
  const uint8_t* act_scales;  // tiled e4m3, rows padded to 256
  const uint8_t* w_scales;    // tiled e4m3, rows padded to 256
  const uint16_t* bias;       // bf16 [N] or null
  float alpha;                // s_a * s_w
  int* dev_status;            // may be null
  unsigned long long timeout_ns;
  GeluQuantParams gq;         // used by the GELU-MLP epilogue only
  QkvParams qk;               // used by the QKV epilogue only
  FusedQuantParams fq;        // used by the fused layer kernel only
  const float* row_factor;    // fp16-operand (INT4) kernel: y = bf16(D f_row[m] f_col[n] + b)
  const float* col_factor;
};

struct GemmTmaps {
  CUtensorMap a, b, la, lb, y;
};

cudaError_t launch_gemm_nvfp4(const GemmNvfp4Params& p, const GemmTmaps& t, int num_sms, cudaStream_t stream,
                              bool pdl);
// Same mainloop, GELU-MLP epilogue (t.y unused).
cudaError_t launch_gemm_nvfp4_gelu(const GemmNvfp4Params& p, const GemmTmaps& t, int num_sms, cudaStream_t stream,
                                   bool pdl);
// Same mainloop, QKV + RMSNorm + RoPE epilogue (t.y unused).
cudaError_t launch_gemm_nvfp4_qkv(const GemmNvfp4Params& p, const GemmTmaps& t, int num_sms, cudaStream_t stream,
                                  bool pdl);
// lora_act bf16 [M, 64] = [hi | lo] of u_work [M, 32] * lora_scale.
cudaError_t launch_lowrank_finalize(const float* u_work, int M, float lora_scale, uint16_t* lora_act,
                                    cudaStream_t stream, bool pdl);

// The CTA-pair kernel: B and [L2^T|L2^T] boxes are 128 rows (half a tile),
// block scales are read through 2D maps of 256-byte rows (box 256 x 8).
struct GemmPairTmaps {
  CUtensorMap a, b, la, lb, y, sfa, sfb;
};

cudaError_t launch_gemm_nvfp4_pair(const GemmNvfp4Params& p, const GemmPairTmaps& t, cudaStream_t stream, bool pdl);
cudaError_t launch_gemm_nvfp4_pair_gelu(const GemmNvfp4Params& p, const GemmPairTmaps& t, cudaStream_t stream,
                                        bool pdl);
cudaError_t launch_gemm_nvfp4_pair_qkv(const GemmNvfp4Params& p, const GemmPairTmaps& t, cudaStream_t stream,
                                       bool pdl);
// The INT4 product on fp16 operands (dequant_int4.cu): t.a / t.b map the fp16
// [M, K] / [N, K] operands as bytes (128-byte boxes of 64 elements), t.la /
// t.lb the scaled low-rank operands; t.sfa / t.sfb are unused.
cudaError_t launch_gemm_f16_pair(const GemmNvfp4Params& p, const GemmPairTmaps& t, cudaStream_t stream, bool pdl);
// The fused layer kernel (p.fq set; t.a / t.sfa / t.la map the buffers the
// kernel itself fills).  tm_x maps x [M, K] bf16 and tm_l1 L1^T [32, K] fp16,
// both in 64 x 128 / 64 x 32 SWIZZLE_128B boxes (the quantizer's chunks).
cudaError_t launch_layer_nvfp4_pair(const GemmNvfp4Params& p, const GemmPairTmaps& t, const CUtensorMap& tm_x,
                                    const CUtensorMap& tm_l1, cudaStream_t stream, bool pdl);

size_t dequant_int4_smem_bytes(int K);
// One launch for both operands (pw: weight rows, pa: activation rows; same K).
cudaError_t launch_dequant_int4(const DequantInt4Params& pw, const DequantInt4Params& pa, cudaStream_t stream,
                                bool pdl);

// The INT4 layer's product with the fp16 operands built inside the GEMM
// (gemm_int4_pair.cu): a4 / b4 map the packed codes [M, K/2] / [N, K/2] in
// 32-byte x 128-row boxes, la / lb the scaled low-rank operands (bf16
// [rows, 64], 64 x 128 SWIZZLE_128B boxes), y the output (16 x 32 boxes,
// 32-byte swizzle).
struct GemmInt4DqParams {
  int M, N, K, M_pad, N_pad;
  const uint16_t* act_scales;  // bf16 [K/64][M_pad]
  const uint16_t* w_scales;    // bf16 [K/64][N_pad]
  const uint16_t* bias;        // bf16 [N] or null
  const float* row_factor;     // 2^Ea [M]
  const float* col_factor;     // 2^Ew [N]
  int* dev_status;
  unsigned long long timeout_ns;
};

struct GemmInt4DqTmaps {
  CUtensorMap a4, b4, la, lb, y;
};

cudaError_t launch_gemm_int4_pair(const GemmInt4DqParams& p, const GemmInt4DqTmaps& t, cudaStream_t stream,
                                  bool pdl);

struct GemmInt4Params {
  int M, N, K, M_pad, N_pad;
  const uint16_t* act_scales;  // bf16 [K/64][M_pad]
  const uint16_t* w_scales;    // bf16 [K/64][N_pad]
  const uint16_t* bias;        // bf16 [N] or null
  uint16_t* y;                 // bf16 [M, N]
  int* dev_status;
  unsigned long long timeout_ns;
};

struct GemmInt4Tmaps {
  CUtensorMap a, b, la, lb;
};

cudaError_t launch_gemm_int4(const GemmInt4Params& p, const GemmInt4Tmaps& t, int num_sms, cudaStream_t stream,
                             bool pdl);

struct AwqParams {
  int M, N, K;
  const uint16_t* x;       // bf16 [M, K]
  const uint8_t* qweight;  // [N, K/2]
  const uint16_t* scales;  // bf16 [N, K/64]
  const uint8_t* zeros;    // [N, K/128] two 4-bit zeros per byte
  const uint16_t* bias;    // bf16 [N] or null
  uint16_t* y;             // bf16 [M, N]
};

cudaError_t launch_awq(const AwqParams& p, int num_sms, cudaStream_t stream, bool pdl);

// Records a message for svdq_last_error() and returns `status`.
int record_error(int status, const char* fmt, ...);

// Unique id (cuCtxGetId) of the calling thread's current CUDA context, or 0
// when no context is current or the driver cannot tell.  Ids are never
// reused within a process, so a device address cached under one id is
// known to be stale once the id changes (for example after cudaDeviceReset).
unsigned long long current_context_id();

// Tensor-map encoding through the driver entry point (no libcuda link needed).
bool encode_tmap_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
                    uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz);

}  // namespace svdq
