// Exact fp16 values of INT4 codes times their bf16 group scale, shared by the
// kernels that build the INT4 layer's fp16 operands (dequant_int4.cu,
// quantize_act.cu in its layer mode, gemm_int4_pair.cu).
//
// Pages: "Nunchaku Lite" docs, "Supported quantization types" table
// (svdq_w4a4, int4, group 64).  A bf16 scale carries 8 significant bits and a
// code |q| <= 8 at most 3, so s q has at most 11: exact in fp16 once the row
// is scaled by a power of two that keeps its largest value below 2^16:
//
//   E[r] = floor(log2(max_g s[r,g])) - 12, clamped to [-100, 100] (0 for a
//          row whose scales are all zero),
//
// and then exact for every group within 2^29 of the row's largest scale
// (smaller groups round as fp16 subnormals), as long as the clamp is not
// reached: a row whose largest scale is 2^113 or more keeps E = 100 and its
// largest values leave fp16's range.  Within every 8-code word the
// values come out in the order (0, 2, 4, 6, 1, 3, 5, 7); every kernel that
// writes an operand uses this order for both operands of the product.
#pragma once
#include <cstdint>

#include "ptx.cuh"

namespace svdq {

SVDQ_DEV uint32_t i4_prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}
SVDQ_DEV uint32_t i4_hsub2_rn(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
SVDQ_DEV uint32_t i4_hmul2_rn(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
// fp32 -> the same fp16 in both halves (round to nearest even).
SVDQ_DEV uint32_t i4_f16x2_dup(float v) {
  uint32_t d;
  asm("cvt.rn.f16x2.f32 %0, %1, %1;" : "=r"(d) : "f"(v));
  return d;
}
// 2^e as an fp32 bit pattern, -126 <= e <= 127.
SVDQ_DEV float i4_exp2i(int e) { return __int_as_float((e + 127) << 23); }

// E of a row from its largest group scale (fp32 value of a bf16 scale).
SVDQ_DEV int i4_row_exponent(float max_scale) {
  if (!(max_scale > 0.f)) return 0;
  const int biased = (__float_as_int(max_scale) >> 23) & 0xFF;   // 0 for an fp32 subnormal
  const int e = (biased == 0 ? -126 : biased - 127) - 12;
  return e < -100 ? -100 : (e > 100 ? 100 : e);
}

// Eight codes (one word, code 2j in the low nibble of byte j) times the
// f16x2 scale s2 -> 16 bytes of fp16 in the order (0,2), (4,6), (1,3), (5,7):
// the code's bits with bit 3 flipped (q + 8) in the low byte of the fp16
// pattern of 1024 (whose unit in the last place is 1), minus 1032, leave q
// exactly; one fp16 multiply by the scale gives the value.
SVDQ_DEV uint4 i4_dequant_word(uint32_t w, uint32_t s2) {
  w ^= 0x88888888u;
  const uint32_t lo = w & 0x0F0F0F0Fu, hi = (w >> 4) & 0x0F0F0F0Fu;
  constexpr uint32_t kMagic = 0x64646464u;   // high byte of the fp16 pattern of 1024
  constexpr uint32_t kBias = 0x64086408u;    // 1032 in both halves
  return make_uint4(i4_hmul2_rn(i4_hsub2_rn(i4_prmt(lo, kMagic, 0x4140u), kBias), s2),
                    i4_hmul2_rn(i4_hsub2_rn(i4_prmt(lo, kMagic, 0x4342u), kBias), s2),
                    i4_hmul2_rn(i4_hsub2_rn(i4_prmt(hi, kMagic, 0x4140u), kBias), s2),
                    i4_hmul2_rn(i4_hsub2_rn(i4_prmt(hi, kMagic, 0x4342u), kBias), s2));
}

}  // namespace svdq
