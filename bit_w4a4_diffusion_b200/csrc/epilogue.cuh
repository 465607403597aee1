// Device helpers of the fused GEMM epilogues (the GELU-MLP epilogue's GELU,
// quantizer staging and low-rank partial products; shared-memory vector
// access), used by both NVFP4 GEMM kernels.
#pragma once
#include <cuda_fp16.h>
#include <cstdint>

#include "ptx.cuh"

namespace svdq {

SVDQ_DEV float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

SVDQ_DEV float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// GELU(v) = v Phi(v) with Phi the standard normal CDF (the exact erf form),
// Phi(-|v|) = erfc(|v| / sqrt 2) / 2 taken from Abramowitz & Stegun,
// "Handbook of Mathematical Functions", formula 7.1.26 (Hastings):
//   erfc(x) ~ (a1 t + a2 t^2 + a3 t^3 + a4 t^4 + a5 t^5) exp(-x^2),
//   t = 1 / (1 + p x),  x >= 0,  absolute error <= 1.5e-7,
// evaluated with the hardware reciprocal and base-2 exponential.  Taking
// Phi(v) = erfc/2 for v < 0 and 1 - erfc/2 for v >= 0 keeps the small
// negative tail free of cancellation.
// Two elements at a time on the packed fp32x2 pipe (each lane of a packed
// operation rounds like its scalar counterpart).
SVDQ_DEV float2 f2(float a) { return make_float2(a, a); }
SVDQ_DEV float2 gelu2(float2 v) {
  const float2 x = __fmul2_rn(make_float2(fabsf(v.x), fabsf(v.y)), f2(0.70710678118654752f));
  const float2 den = __ffma2_rn(f2(0.3275911f), x, f2(1.0f));
  const float2 t = make_float2(rcp_approx(den.x), rcp_approx(den.y));
  float2 q = __ffma2_rn(f2(1.061405429f), t, f2(-1.453152027f));
  q = __ffma2_rn(q, t, f2(1.421413741f));
  q = __ffma2_rn(q, t, f2(-0.284496736f));
  q = __ffma2_rn(q, t, f2(0.254829592f));
  q = __fmul2_rn(q, t);
  const float2 arg = __fmul2_rn(__fmul2_rn(x, x), f2(-1.4426950408889634f));  // -x^2 log2(e)
  const float2 e = make_float2(ex2_approx(arg.x), ex2_approx(arg.y));         // exp(-x^2)
  const float2 half_erfc = __fmul2_rn(__fmul2_rn(f2(0.5f), q), e);
  const float2 upper = __fadd2_rn(f2(1.0f), make_float2(-half_erfc.x, -half_erfc.y));
  const float2 phi = make_float2(v.x < 0.f ? half_erfc.x : upper.x, v.y < 0.f ? half_erfc.y : upper.y);
  return __fmul2_rn(v, phi);
}

SVDQ_DEV uint32_t half2_bits(float lo, float hi) {
  uint32_t out;
  asm("cvt.rn.f16x2.f32 %0, %2, %1;" : "=r"(out) : "f"(lo), "f"(hi));
  return out;  // lo in the low half
}

SVDQ_DEV void st_shared_v4(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

// D (fp32) += A (16 x 16 fp16, row) * B (16 x 8 fp16, col).
SVDQ_DEV void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                        uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

SVDQ_DEV void red_add_f32x2(float* addr, float a, float b) {
  asm volatile("red.global.add.v2.f32 [%0], {%1, %2};" ::"l"(addr), "f"(a), "f"(b) : "memory");
}

// Byte offset of scale (row, group) in the tiled NVFP4 scale layout.
SVDQ_DEV size_t tiled_scale_offset(int row, int group, int K) {
  return ((size_t)(row >> 7) * (K / 64) + (group >> 2)) * 512 + (row & 31) * 16 + ((row & 127) >> 5) * 4 + (group & 3);
}

// 16-byte segment s (fp16 columns 8s..8s+7) of row r in a warp's 32 x 16
// fp16 staging tile (32-byte rows; segments XOR-ed with (r / 4) mod 2 so that
// both the row-per-lane stores and the fragment loads are conflict-free).
SVDQ_DEV uint32_t hseg16(uint32_t base, int r, int s) {
  return base + (uint32_t)r * 32u + (uint32_t)((s ^ ((r >> 2) & 1)) << 4);
}

SVDQ_DEV uint4 ld_shared_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr)
               : "memory");
  return v;
}

SVDQ_DEV uint2 ld_shared_v2(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr) : "memory");
  return v;
}

}  // namespace svdq
