// The INT4 product on the fp16 tensor pipe: exact fp16 operands from the
// 4-bit codes and their bf16 group scales.
//
// Pages: "Nunchaku Lite" docs, "Supported quantization types" table
// (svdq_w4a4, int4, group 64) and its tip that int4 checkpoints on Blackwell
// may be slower than nvfp4: these tensor cores have no 4-bit integer MMA.
// What the layer needs from the INT4 residual branch is
//
//   sum_g sa[m,g] sw[n,g] sum_{k in g} qa[m,k] qw[n,k]  =  sum_k A[m,k] W[n,k],
//   A[m,k] = sa[m,k/64] qa[m,k],   W[n,k] = sw[n,k/64] qw[n,k],
//
// and each dequantized value is exact in fp16: a bf16 scale carries 8
// significant bits and a code |q| <= 8 at most 3, so their product has at
// most 11, which is fp16's precision.  fp16's exponent range is narrower than
// bf16's, so row r is scaled by a power of two chosen from its largest scale:
//
//   E[r]      = floor(log2(max_g s[r,g])) - 12, clamped to [-100, 100]
//               (0 for a row whose scales are all zero)
//   out[r,k]  = fp16(s[r,k/64] 2^-E[r] q[r,k])   exact whenever
//               s[r,g] >= 2^(E[r] - 17), i.e. for every group within 2^29 of
//               the row's largest scale (smaller groups round as fp16
//               subnormals, an error below 2^-36 of the row's largest value);
//               the largest is below 8 * 2^13 = 65536, within fp16's 65504
//               since a scale's significand is at most 255/128
//   lora[r,:] = lora_in[r,:] 2^-E[r]        (bf16, exact)
//   f[r]      = 2^E[r]                       (fp32)
//
// so that the GEMM's fp32 sum D[m,n] = sum_k out_a[m,k] out_w[n,k] + lora_a .
// lora_w equals the layer's sum times 2^-(E_a[m] + E_w[n]), undone in its
// epilogue by f_a[m] f_w[n].
//
// Order along K: within every 8-code word the outputs are stored as
// elements (0, 2, 4, 6, 1, 3, 5, 7) -- the order in which the low and then
// the high nibbles of the word's four bytes come out of the conversion.  Both
// operands of the product are stored in this order, so every dot product
// pairs the same elements as in natural order, and a word never straddles a
// 64-group.
//
// Conversion of a code: the code's bits with bit 3 flipped are q + 8 in
// 0..15; placed in the low byte of the fp16 pattern 0x6400 (1024, whose unit
// in the last place is 1) they give 1024 + q + 8, and subtracting 1032 leaves
// q exactly; one fp16 multiply by the scaled group scale gives the value
// (exact, see above).  Two codes per packed f16x2 operation.
//
// One CTA of 256 threads per 16 rows: the rows' scales are staged in shared
// memory (group-major, so a group's 16 row scales are one 32-byte read), the
// row exponents come from them, then each thread turns 16 bytes of codes into
// 64 bytes of fp16 at a time, consecutive threads along a row (coalesced).
#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"
#include "svdq_internal.h"

namespace svdq {
namespace {

constexpr int DQ_ROWS = 16;
constexpr int DQ_THREADS = 256;

SVDQ_DEV uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}
SVDQ_DEV uint32_t hsub2_rn(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
SVDQ_DEV uint32_t hmul2_rn(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
SVDQ_DEV uint32_t f32_to_f16x2_dup(float v) {
  uint32_t d;
  asm("cvt.rn.f16x2.f32 %0, %1, %1;" : "=r"(d) : "f"(v));
  return d;
}
// 2^e as an fp32 bit pattern, -126 <= e <= 127.
SVDQ_DEV float exp2i(int e) { return __int_as_float((e + 127) << 23); }

// Eight codes (one 32-bit word, code 2j in the low nibble of byte j) times
// the f16x2 scale s2 -> four f16x2 words in the order (0,2), (4,6), (1,3), (5,7).
SVDQ_DEV void dequant_word(uint32_t w, uint32_t s2, uint32_t (&o)[4]) {
  w ^= 0x88888888u;                          // q + 8 in every nibble
  const uint32_t lo = w & 0x0F0F0F0Fu;       // codes 0, 2, 4, 6 (one per byte)
  const uint32_t hi = (w >> 4) & 0x0F0F0F0Fu;  // codes 1, 3, 5, 7
  constexpr uint32_t kMagic = 0x64646464u;   // high byte of the fp16 pattern of 1024
  constexpr uint32_t kBias = 0x64086408u;    // 1032 in both halves
  o[0] = hmul2_rn(hsub2_rn(prmt(lo, kMagic, 0x4140u), kBias), s2);
  o[1] = hmul2_rn(hsub2_rn(prmt(lo, kMagic, 0x4342u), kBias), s2);
  o[2] = hmul2_rn(hsub2_rn(prmt(hi, kMagic, 0x4140u), kBias), s2);
  o[3] = hmul2_rn(hsub2_rn(prmt(hi, kMagic, 0x4342u), kBias), s2);
}

__global__ void __launch_bounds__(DQ_THREADS) dequant_int4_kernel(DequantInt4Params p) {
  extern __shared__ float dq_smem[];
  const int groups = p.K / 64;
  float* sc = dq_smem;                          // [groups][DQ_ROWS]
  float* inv = dq_smem + groups * DQ_ROWS;      // [DQ_ROWS]: 2^-E[r]
  const int r0 = blockIdx.x * DQ_ROWS;
  const int tid = threadIdx.x;
  pdl_wait();
  pdl_launch_dependents();

  // Scales of the CTA's rows (rows past R read the zero padding: R_pad is a
  // multiple of 256 and r0 + DQ_ROWS <= R_pad).
  for (int i = tid; i < groups * DQ_ROWS; i += DQ_THREADS) {
    const int g = i / DQ_ROWS, r = i - g * DQ_ROWS;
    sc[i] = __bfloat162float(__ushort_as_bfloat16(p.scales[(size_t)g * p.R_pad + r0 + r]));
  }
  __syncthreads();
  if (tid < DQ_ROWS) {
    float mx = 0.f;
    for (int g = 0; g < groups; ++g) mx = fmaxf(mx, sc[g * DQ_ROWS + tid]);
    int e = 0;
    if (mx > 0.f) {
      const int biased = (__float_as_int(mx) >> 23) & 0xFF;   // 0 for an fp32 subnormal
      e = (biased == 0 ? -126 : biased - 127) - 12;
      e = e < -100 ? -100 : (e > 100 ? 100 : e);
    }
    inv[tid] = exp2i(-e);
    if (r0 + tid < p.R) p.factor[r0 + tid] = exp2i(e);
  }
  __syncthreads();

  // Codes: 16 bytes (32 codes, all in one 64-group) per step.
  const int chunks = p.K / 32;
  for (int i = tid; i < DQ_ROWS * chunks; i += DQ_THREADS) {
    const int r = i / chunks, j = i - r * chunks;
    const int row = r0 + r;
    if (row >= p.R) break;   // rows are visited in order: the rest are past R too
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(p.codes + (size_t)row * (p.K / 2)) + j);
    // The scaled group scale: exact in fp32 (a power-of-two factor), then in
    // fp16 for every group within 2^29 of the row's largest.
    const uint32_t s2 = f32_to_f16x2_dup(__fmul_rn(sc[(j >> 1) * DQ_ROWS + r], inv[r]));
    uint32_t o[4][4];
    dequant_word(w.x, s2, o[0]);
    dequant_word(w.y, s2, o[1]);
    dequant_word(w.z, s2, o[2]);
    dequant_word(w.w, s2, o[3]);
    uint4* dst = reinterpret_cast<uint4*>(p.out + (size_t)row * p.K) + 4 * j;
#pragma unroll
    for (int q = 0; q < 4; ++q) dst[q] = make_uint4(o[q][0], o[q][1], o[q][2], o[q][3]);
  }

  // The low-rank operand rows, scaled by the same power of two.
  if (p.lora_in != nullptr) {
    for (int i = tid; i < DQ_ROWS * 64; i += DQ_THREADS) {
      const int r = i >> 6, c = i & 63;
      const int row = r0 + r;
      if (row >= p.R) break;
      const float v = __bfloat162float(__ushort_as_bfloat16(p.lora_in[(size_t)row * 64 + c]));
      p.lora_out[(size_t)row * 64 + c] = __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(v, inv[r])));
    }
  }
}

}  // namespace

size_t dequant_int4_smem_bytes(int K) { return (size_t)((K / 64) * DQ_ROWS + DQ_ROWS) * sizeof(float); }

cudaError_t launch_dequant_int4(const DequantInt4Params& p, cudaStream_t stream, bool pdl) {
  const size_t smem = dequant_int4_smem_bytes(p.K);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(dequant_int4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((p.R + DQ_ROWS - 1) / DQ_ROWS));
  cfg.blockDim = dim3(DQ_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  set_pdl(cfg, attr, pdl);
  return cudaLaunchKernelEx(&cfg, dequant_int4_kernel, p);
}

}  // namespace svdq
