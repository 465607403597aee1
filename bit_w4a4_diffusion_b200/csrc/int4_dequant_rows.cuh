// One block's share of the INT4 operand pass (dequant_int4.cu): kRows rows
// of a [R, K] INT4 matrix turned into the layer's fp16 operand rows, their
// powers of two and their scaled low-rank rows (int4_fp16.cuh for the
// arithmetic).  Used by the operand-pass kernel and by the extra blocks of
// the INT4 quantizer's launch that convert the weight rows beside it.
//
// kRows * 16 threads, 16 per row: thread (r, l) takes the 16-byte code chunks
// l, l + 16, ... of row r (a row's 16 threads read 256 contiguous bytes per
// step), issuing the loads of up to eight chunks before it converts any.  The
// rows' scales are staged in `sc` (shared, (K/64) * kRows floats,
// group-major so that a group's row scales are one contiguous read) and a
// row's largest scale is a max over its 16 threads.  Every thread of the
// block calls it (it contains block barriers).
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "int4_fp16.cuh"
#include "ptx.cuh"
#include "svdq_internal.h"

namespace svdq {

constexpr int kDqThreadsPerRow = 16;
constexpr int kDqBatch = 8;   // chunk loads in flight per thread

template <int kRows>
__device__ __forceinline__ void int4_dequant_rows(const DequantInt4Params& p, int r0, float* sc) {
  constexpr int kThreads = kRows * kDqThreadsPerRow;
  const int groups = p.K / 64;
  const int tid = threadIdx.x;
  const int r = tid / kDqThreadsPerRow, l = tid % kDqThreadsPerRow;
  const int row = r0 + r;
  const bool row_ok = row < p.R;

  // Scales of the block's rows (rows past R read the zero padding: R_pad is
  // a multiple of 256 and r0 + kRows <= R_pad).  The first barrier ends the
  // previous call's reads of `sc`.
  __syncthreads();
  for (int i = tid; i < groups * kRows; i += kThreads) {
    const int g = i / kRows, rr = i - g * kRows;
    sc[i] = __bfloat162float(__ushort_as_bfloat16(p.scales[(size_t)g * p.R_pad + r0 + rr]));
  }
  __syncthreads();
  float mx = 0.f;
  for (int g = l; g < groups; g += kDqThreadsPerRow) mx = fmaxf(mx, sc[g * kRows + r]);
#pragma unroll
  for (int o = kDqThreadsPerRow / 2; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  const int e = i4_row_exponent(mx);
  const float inv = i4_exp2i(-e);
  if (row_ok && l == 0) p.factor[row] = i4_exp2i(e);

  if (row_ok && p.out != nullptr) {
    // Codes: 16 bytes (32 codes, all in one 64-group) per chunk.
    const int chunks = p.K / 32;
    const uint4* src = reinterpret_cast<const uint4*>(p.codes + (size_t)row * (p.K / 2));
    uint4* dst = reinterpret_cast<uint4*>(p.out + (size_t)row * p.K);
    for (int j0 = l; j0 < chunks; j0 += kDqThreadsPerRow * kDqBatch) {
      uint4 w[kDqBatch];
#pragma unroll
      for (int b = 0; b < kDqBatch; ++b) {
        const int j = j0 + kDqThreadsPerRow * b;
        if (j < chunks) w[b] = __ldg(src + j);
      }
#pragma unroll
      for (int b = 0; b < kDqBatch; ++b) {
        const int j = j0 + kDqThreadsPerRow * b;
        if (j < chunks) {
          // The scaled group scale: exact in fp32 (a power-of-two factor),
          // then in fp16 for every group within 2^29 of the row's largest.
          const uint32_t s2 = i4_f16x2_dup(__fmul_rn(sc[(j >> 1) * kRows + r], inv));
          dst[4 * j] = i4_dequant_word(w[b].x, s2);
          dst[4 * j + 1] = i4_dequant_word(w[b].y, s2);
          dst[4 * j + 2] = i4_dequant_word(w[b].z, s2);
          dst[4 * j + 3] = i4_dequant_word(w[b].w, s2);
        }
      }
    }
  }
  if (row_ok && p.lora_in != nullptr) {
    // The low-rank operand row, scaled by the same power of two: four values
    // per thread.
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

}  // namespace svdq
