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
// The conversion of a code and the order of the values within every 8 codes,
// (0, 2, 4, 6, 1, 3, 5, 7) for both operands of the product, are those of
// int4_fp16.cuh.
//
// One launch converts both operands (the weight rows first, then the
// activation rows: one grid, so the two passes share a single ramp-up and
// tail).  One CTA of 128 threads per 8 rows, 16 threads per row: thread (r, l)
// takes the 16-byte code chunks l, l + 16, l + 32, ... of row r (a row's 16
// threads read 256 contiguous bytes per step), issuing the loads of up to
// eight chunks before it converts any, so that enough bytes are in flight to
// cover the memory latency.  The rows' scales are staged in shared memory
// (group-major, so a group's 8 row scales are one 16-byte read) and each
// row's largest scale is a max over its 16 threads.
#include <cuda_bf16.h>
#include <cstdint>

#include "int4_fp16.cuh"
#include "ptx.cuh"
#include "svdq_internal.h"

namespace svdq {
namespace {

constexpr int DQ_ROWS = 8;
constexpr int DQ_TPR = 16;                         // threads per row
constexpr int DQ_THREADS = DQ_ROWS * DQ_TPR;
constexpr int DQ_BATCH = 8;                        // chunk loads in flight per thread

__global__ void __launch_bounds__(DQ_THREADS) dequant_int4_kernel(DequantInt4Params pw, DequantInt4Params pa) {
  extern __shared__ float dq_smem[];
  const int blocks_w = (pw.R + DQ_ROWS - 1) / DQ_ROWS;
  const bool is_w = (int)blockIdx.x < blocks_w;
  const DequantInt4Params p = is_w ? pw : pa;
  const int groups = p.K / 64;
  float* sc = dq_smem;                          // [groups][DQ_ROWS]
  const int r0 = ((int)blockIdx.x - (is_w ? 0 : blocks_w)) * DQ_ROWS;
  const int tid = threadIdx.x;
  const int r = tid / DQ_TPR, l = tid % DQ_TPR;
  const int row = r0 + r;
  const bool row_ok = row < p.R;
  pdl_wait();
  pdl_launch_dependents();

  // Scales of the CTA's rows (rows past R read the zero padding: R_pad is a
  // multiple of 256 and r0 + DQ_ROWS <= R_pad).
  for (int i = tid; i < groups * DQ_ROWS; i += DQ_THREADS) {
    const int g = i / DQ_ROWS, rr = i - g * DQ_ROWS;
    sc[i] = __bfloat162float(__ushort_as_bfloat16(p.scales[(size_t)g * p.R_pad + r0 + rr]));
  }
  __syncthreads();
  // The row's largest scale: each of its 16 threads takes every 16th group.
  float mx = 0.f;
  for (int g = l; g < groups; g += DQ_TPR) mx = fmaxf(mx, sc[g * DQ_ROWS + r]);
#pragma unroll
  for (int o = DQ_TPR / 2; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  const int e = i4_row_exponent(mx);
  const float inv = i4_exp2i(-e);
  if (row_ok && l == 0) p.factor[row] = i4_exp2i(e);

  if (row_ok && p.out != nullptr) {
    // Codes: 16 bytes (32 codes, all in one 64-group) per chunk.
    const int chunks = p.K / 32;
    const uint4* src = reinterpret_cast<const uint4*>(p.codes + (size_t)row * (p.K / 2));
    uint4* dst = reinterpret_cast<uint4*>(p.out + (size_t)row * p.K);
    for (int j0 = l; j0 < chunks; j0 += DQ_TPR * DQ_BATCH) {
      uint4 w[DQ_BATCH];
#pragma unroll
      for (int b = 0; b < DQ_BATCH; ++b) {
        const int j = j0 + DQ_TPR * b;
        if (j < chunks) w[b] = __ldg(src + j);
      }
#pragma unroll
      for (int b = 0; b < DQ_BATCH; ++b) {
        const int j = j0 + DQ_TPR * b;
        if (j < chunks) {
          // The scaled group scale: exact in fp32 (a power-of-two factor),
          // then in fp16 for every group within 2^29 of the row's largest.
          const uint32_t s2 = i4_f16x2_dup(__fmul_rn(sc[(j >> 1) * DQ_ROWS + r], inv));
          dst[4 * j] = i4_dequant_word(w[b].x, s2);
          dst[4 * j + 1] = i4_dequant_word(w[b].y, s2);
          dst[4 * j + 2] = i4_dequant_word(w[b].z, s2);
          dst[4 * j + 3] = i4_dequant_word(w[b].w, s2);
        }
      }
    }
  }
  if (row_ok) {
    // The low-rank operand row, scaled by the same power of two: four
    // values per thread.
    if (p.lora_in != nullptr) {
      const uint2 v = __ldg(reinterpret_cast<const uint2*>(p.lora_in + (size_t)row * 64) + l);
      auto scale2 = [&](uint32_t b) {
        const float lo = __fmul_rn(__uint_as_float(b << 16), inv);
        const float hi = __fmul_rn(__uint_as_float(b & 0xFFFF0000u), inv);
        return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(lo)) |
               ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(hi)) << 16);
      };
      reinterpret_cast<uint2*>(p.lora_out + (size_t)row * 64)[l] = make_uint2(scale2(v.x), scale2(v.y));
    }
  }
}

}  // namespace

size_t dequant_int4_smem_bytes(int K) { return (size_t)(K / 64) * DQ_ROWS * sizeof(float); }

cudaError_t launch_dequant_int4(const DequantInt4Params& pw, const DequantInt4Params& pa, cudaStream_t stream,
                                bool pdl) {
  const size_t smem = dequant_int4_smem_bytes(pw.K);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(dequant_int4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((pw.R + DQ_ROWS - 1) / DQ_ROWS + (pa.R + DQ_ROWS - 1) / DQ_ROWS));
  cfg.blockDim = dim3(DQ_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  set_pdl(cfg, attr, pdl);
  return cudaLaunchKernelEx(&cfg, dequant_int4_kernel, pw, pa);
}

}  // namespace svdq
