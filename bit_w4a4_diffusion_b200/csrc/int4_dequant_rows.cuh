// One block's share of the INT4 operand pass (dequant_int4.cu): kRows rows
// of a [R, K] INT4 matrix turned into the layer's fp16 operand rows, their
// powers of two and their scaled low-rank rows (int4_fp16.cuh for the
// arithmetic).  Used by the operand-pass kernel and by the extra blocks of
// the INT4 quantizer's launch that convert the weight rows beside it.
//
// kRows * 16 threads, 16 per row.  The rows' scales are staged in shared
// memory (group-major, so that a group's row scales are one contiguous read)
// and a row's largest scale is a max over its 16 threads.  The codes go
// through shared memory too, kDqChunkWords 4-byte words (8 codes each) of
// every row at a time: the block loads them with 16-byte loads, then thread
// (r, l) converts words l, l + 16, ... of row r, so that each store
// instruction writes 256 contiguous bytes of a row (one 16-byte fp16 group
// of 8 values per thread).  Converting a whole 16-byte chunk per thread
// instead leaves every store 64 bytes apart from its neighbour's, which
// writes each 32-byte sector in two halves.  Every thread of the block calls
// it (it contains block barriers).
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "int4_fp16.cuh"
#include "ptx.cuh"
#include "svdq_internal.h"

namespace svdq {

constexpr int kDqThreadsPerRow = 16;
constexpr int kDqChunkWords = 384;                      // 3072 codes of a row per staging round
constexpr int kDqStageStride = kDqChunkWords + 16;      // words; rows r, r + 1 land 16 banks apart

// Shared memory the routine needs for kRows rows of length K.
__host__ __device__ constexpr size_t int4_dequant_rows_smem(int rows, int K) {
  return (size_t)(K / 64) * rows * sizeof(float) + (size_t)rows * kDqStageStride * sizeof(uint32_t);
}

template <int kRows>
__device__ __forceinline__ void int4_dequant_rows(const DequantInt4Params& p, int r0, float* smem) {
  constexpr int kThreads = kRows * kDqThreadsPerRow;
  const int groups = p.K / 64;
  float* sc = smem;                                                   // [groups][kRows]
  uint32_t* stage = reinterpret_cast<uint32_t*>(smem + groups * kRows);   // [kRows][kDqStageStride]
  const int tid = threadIdx.x;
  const int r = tid / kDqThreadsPerRow, l = tid % kDqThreadsPerRow;
  const int row = r0 + r;
  const bool row_ok = row < p.R;

  // Scales of the block's rows (rows past R read the zero padding: R_pad is
  // a multiple of 256 and r0 + kRows <= R_pad).  The first barrier ends the
  // previous call's reads of shared memory.
  __syncthreads();
  for (int i = tid; i < groups * kRows; i += kThreads) {
    const int g = i / kRows, rr = i - g * kRows;
    sc[i] = __bfloat162float(__ushort_as_bfloat16(p.scales[(size_t)g * p.R_pad + r0 + rr]));
  }
  // The low-rank operand row is read now, ahead of the stores below.
  uint2 lora = make_uint2(0, 0);
  if (row_ok && p.lora_in != nullptr) lora = __ldg(reinterpret_cast<const uint2*>(p.lora_in + (size_t)row * 64) + l);
  __syncthreads();
  float mx = 0.f;
  for (int g = l; g < groups; g += kDqThreadsPerRow) mx = fmaxf(mx, sc[g * kRows + r]);
#pragma unroll
  for (int o = kDqThreadsPerRow / 2; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  const int e = i4_row_exponent(mx);
  const float inv = i4_exp2i(-e);
  if (row_ok && l == 0) p.factor[row] = i4_exp2i(e);

  if (p.out != nullptr) {
    const int words = p.K / 8;   // a multiple of 32 (K % 256 == 0)
    for (int w0 = 0; w0 < words; w0 += kDqChunkWords) {
      const int nw = words - w0 < kDqChunkWords ? words - w0 : kDqChunkWords;
      const int nq = nw / 4;     // 16-byte loads per row
      // The previous round's readers are done with the stage.
      __syncthreads();
      constexpr int kLoads = (kRows * kDqChunkWords / 4 + kThreads - 1) / kThreads;
      uint4 v[kLoads];
#pragma unroll
      for (int b = 0; b < kLoads; ++b) {
        const int i = tid + b * kThreads;
        const int rr = i / nq, c = i - rr * nq;
        if (rr < kRows && r0 + rr < p.R)
          v[b] = __ldg(reinterpret_cast<const uint4*>(p.codes + (size_t)(r0 + rr) * (p.K / 2) + (size_t)w0 * 4) + c);
      }
#pragma unroll
      for (int b = 0; b < kLoads; ++b) {
        const int i = tid + b * kThreads;
        const int rr = i / nq, c = i - rr * nq;
        if (rr < kRows && r0 + rr < p.R) *reinterpret_cast<uint4*>(stage + rr * kDqStageStride + 4 * c) = v[b];
      }
      __syncthreads();
      if (row_ok) {
        uint4* dst = reinterpret_cast<uint4*>(p.out + (size_t)row * p.K) + w0;
        for (int w = l; w < nw; w += kDqThreadsPerRow) {
          // The scaled group scale: exact in fp32 (a power-of-two factor),
          // then in fp16 for every group within 2^29 of the row's largest.
          const uint32_t s2 = i4_f16x2_dup(__fmul_rn(sc[((w0 + w) >> 3) * kRows + r], inv));
          dst[w] = i4_dequant_word(stage[r * kDqStageStride + w], s2);
        }
      }
    }
  }
  if (row_ok && p.lora_in != nullptr) {
    // The low-rank operand row, scaled by the same power of two: four values
    // per thread.
    auto scale2 = [&](uint32_t b) {
      const float lo = __fmul_rn(__uint_as_float(b << 16), inv);
      const float hi = __fmul_rn(__uint_as_float(b & 0xFFFF0000u), inv);
      return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(lo)) |
             ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(hi)) << 16);
    };
    reinterpret_cast<uint2*>(p.lora_out + (size_t)row * 64)[l] = make_uint2(scale2(lora.x), scale2(lora.y));
  }
}

}  // namespace svdq
