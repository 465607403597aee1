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
//               since a scale's significand is at most 255/128.  Both hold
//               while E is not clamped (largest scale in [2^-88, 2^113));
//               beyond 2^113, 8 s 2^-100 leaves fp16's range
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
// tail), 8 rows per 128-thread CTA (int4_dequant_rows.cuh).
#include <cuda_bf16.h>
#include <cstdint>

#include "int4_dequant_rows.cuh"
#include "ptx.cuh"
#include "svdq_internal.h"

namespace svdq {
namespace {

constexpr int DQ_ROWS = 8;
constexpr int DQ_THREADS = DQ_ROWS * kDqThreadsPerRow;

__global__ void __launch_bounds__(DQ_THREADS) dequant_int4_kernel(DequantInt4Params pw, DequantInt4Params pa) {
  extern __shared__ float dq_smem[];   // scales, then the code stage (int4_dequant_rows.cuh)
  const int blocks_w = (pw.R + DQ_ROWS - 1) / DQ_ROWS;
  const bool is_w = (int)blockIdx.x < blocks_w;
  const DequantInt4Params p = is_w ? pw : pa;
  const int r0 = ((int)blockIdx.x - (is_w ? 0 : blocks_w)) * DQ_ROWS;
  pdl_wait();
  pdl_launch_dependents();
  int4_dequant_rows<DQ_ROWS>(p, r0, dq_smem);
}

}  // namespace

size_t dequant_int4_smem_bytes(int K) { return int4_dequant_rows_smem(DQ_ROWS, K); }

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
