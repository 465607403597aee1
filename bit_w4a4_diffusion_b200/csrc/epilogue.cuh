// The fused GEMM epilogues' per-lane arithmetic and its helpers (GELU,
// the down layer's NVFP4 quantizer and low-rank partial products; RMSNorm
// and RoPE of a QKV head; shared-memory vector access), used by both NVFP4
// GEMM kernels.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

#include "ptx.cuh"
#include "svdq_internal.h"

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
// operation rounds like its scalar counterpart).  The polynomial carries the
// 1/2 of Phi = erfc/2 in its coefficients: halving every coefficient halves
// each rounded step exactly, so q below is exactly half the polynomial.
SVDQ_DEV float2 f2(float a) { return make_float2(a, a); }
SVDQ_DEV float2 gelu2(float2 v) {
  const float2 x = __fmul2_rn(make_float2(fabsf(v.x), fabsf(v.y)), f2(0.70710678118654752f));
  const float2 den = __ffma2_rn(f2(0.3275911f), x, f2(1.0f));
  const float2 t = make_float2(rcp_approx(den.x), rcp_approx(den.y));
  float2 q = __ffma2_rn(f2(0.5f * 1.061405429f), t, f2(0.5f * -1.453152027f));
  q = __ffma2_rn(q, t, f2(0.5f * 1.421413741f));
  q = __ffma2_rn(q, t, f2(0.5f * -0.284496736f));
  q = __ffma2_rn(q, t, f2(0.5f * 0.254829592f));
  q = __fmul2_rn(q, t);                                                       // erfc(x) / (2 exp(-x^2))
  const float2 arg = __fmul2_rn(__fmul2_rn(x, x), f2(-1.4426950408889634f));  // -x^2 log2(e)
  const float2 e = make_float2(ex2_approx(arg.x), ex2_approx(arg.y));         // exp(-x^2)
  const float2 half_erfc = __fmul2_rn(q, e);
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

namespace svdq {

// Eight fp32 (four pairs lo, hi) -> four bytes of E2M1 codes, pair i in byte
// i (lo in its low nibble); RNE, satfinite.
SVDQ_DEV uint32_t cvt_e2m1x8(float2 a, float2 b, float2 c, float2 d) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(out)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y), "f"(d.x), "f"(d.y));
  return out;
}

// bf16 pair (the even column in the low half) -> two floats.
SVDQ_DEV float2 bf16x2_to_float2(uint32_t w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

// Per-lane constants of the GELU-MLP epilogue; a lane owns one row of its
// warp's 32 and a warp 32-column chunks of the tile.
struct GeluLane {
  const float* tab_inv;      // the tile's down-layer 1/lambda columns (shared memory)
  const uint16_t* tab_bias;  // the tile's bias columns, bf16 (shared memory)
  float2 alpha2;             // alpha of the up layer, twice
  float2 lr2;                // 2^-e applied before the fp16 conversion, twice
  float inv_six_s;           // fp32(1 / (6 s_d))
  uint32_t hbase;            // the warp's 32 x 16 fp16 staging tile (shared memory)
  int lane, g, c;            // g = lane / 4, c = lane % 4
};

// One 32-column chunk of the GELU-MLP epilogue for the lane's row (tile
// columns cl.., output columns n..; r holds the accumulator, fp32 bits):
//   h_hat = GELU(alpha D + b) * inv_lambda_down   (zero for rows past M)
//   the down layer's NVFP4 codes and scale bytes of the chunk's two groups
//   of 16, stored to gq.codes / gq.scales
//   lacc += the warp's share of fp16(h_hat 2^-e) . L1_down over the chunk,
//           16 columns at a time on mma.sync (lane (g, c) takes fp16 columns
//           4c..4c+3 of the 16 as its k values, a permutation of k shared by
//           both operands)
SVDQ_DEV void gelu_quant_chunk(uint32_t (&r)[32], const GeluLane& L, const GeluQuantParams& gq, int N, int cl, int n,
                               int row, bool row_ok, float (&lacc)[2][4][4]) {
  const int g = L.g, c = L.c;
  // The chunk's low-rank B fragments (from L1 / L2), needed last.
  uint2 bq[2][4];
#pragma unroll
  for (int hh = 0; hh < 2; ++hh)
#pragma unroll
    for (int j = 0; j < 4; ++j)
      bq[hh][j] = __ldg(reinterpret_cast<const uint2*>(gq.l1t + (size_t)(8 * j + g) * N + n + 16 * hh + 4 * c));
  // h_hat in place of the accumulator values.
#pragma unroll
  for (int k8 = 0; k8 < 4; ++k8) {
    const float4 i0v = *reinterpret_cast<const float4*>(L.tab_inv + cl + 8 * k8);
    const float4 i1v = *reinterpret_cast<const float4*>(L.tab_inv + cl + 8 * k8 + 4);
    const uint4 bw = *reinterpret_cast<const uint4*>(L.tab_bias + cl + 8 * k8);
    const uint32_t bb[4] = {bw.x, bw.y, bw.z, bw.w};
    const float il[8] = {i0v.x, i0v.y, i0v.z, i0v.w, i1v.x, i1v.y, i1v.z, i1v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 v = __ffma2_rn(
          L.alpha2, make_float2(__uint_as_float(r[8 * k8 + 2 * j]), __uint_as_float(r[8 * k8 + 2 * j + 1])),
          bf16x2_to_float2(bb[j]));
      const float2 h = __fmul2_rn(gelu2(v), make_float2(il[2 * j], il[2 * j + 1]));
      r[8 * k8 + 2 * j] = __float_as_uint(row_ok ? h.x : 0.f);
      r[8 * k8 + 2 * j + 1] = __float_as_uint(row_ok ? h.y : 0.f);
    }
  }
  // NVFP4 quantization of the two 16-groups (the down layer's rule).
  auto pair = [&](int e, float2 q2) {
    return __fmul2_rn(make_float2(__uint_as_float(r[e]), __uint_as_float(r[e + 1])), q2);
  };
  uint32_t cw[4], sbs = 0;
#pragma unroll
  for (int grp = 0; grp < 2; ++grp) {
    float a = 0.f;
#pragma unroll
    for (int k = 0; k < 16; ++k) a = fmaxf(a, fabsf(__uint_as_float(r[16 * grp + k])));
    const uint32_t sb = cvt_e4m3(__fmul_rn(a, L.inv_six_s));
    const float d = __fmul_rn(e4m3_to_f32(sb), gq.s_d);
    uint32_t w0 = 0, w1 = 0;
    if (d != 0.f) {  // an all-zero group keeps all-zero codes
      const float rr = __frcp_rn(d);
      const float2 q2 = make_float2(rr, rr);
      const int e = 16 * grp;
      w0 = cvt_e2m1x8(pair(e, q2), pair(e + 2, q2), pair(e + 4, q2), pair(e + 6, q2));
      w1 = cvt_e2m1x8(pair(e + 8, q2), pair(e + 10, q2), pair(e + 12, q2), pair(e + 14, q2));
    }
    cw[2 * grp] = w0;
    cw[2 * grp + 1] = w1;
    sbs |= sb << (8 * grp);
  }
  if (row_ok)
    *reinterpret_cast<uint4*>(gq.codes + (size_t)row * (N / 2) + n / 2) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
  *reinterpret_cast<uint16_t*>(gq.scales + tiled_scale_offset(row, n / 16, N)) = (uint16_t)sbs;
  // Low-rank partial, 16 columns at a time.
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
#pragma unroll
    for (int sg = 0; sg < 2; ++sg) {
      uint32_t hv[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 t = pair(16 * hh + 8 * sg + 2 * k, L.lr2);
        hv[k] = half2_bits(t.x, t.y);
      }
      st_shared_v4(hseg16(L.hbase, L.lane, sg), make_uint4(hv[0], hv[1], hv[2], hv[3]));
    }
    __syncwarp();
    uint2 xa[2], xb[2];
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      xa[t] = ld_shared_v2(hseg16(L.hbase, 16 * t + g, c >> 1) + (c & 1) * 8);
      xb[t] = ld_shared_v2(hseg16(L.hbase, 16 * t + 8 + g, c >> 1) + (c & 1) * 8);
    }
    __syncwarp();  // every lane's loads precede the next stores
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int t = 0; t < 2; ++t)
        mma_16816(lacc[t][j], xa[t].x, xb[t].x, xa[t].y, xb[t].y, bq[hh][j].x, bq[hh][j].y);
  }
}

// The QKV epilogue for one lane's row of one 128-feature head (r holds the
// head's accumulator columns, fp32 bits):
//   v = alpha D + b;  for a Q or K head (part 0 / 1) also
//   v * rsqrt(mean(v^2) + eps) * gamma, then each pair (2i, 2i + 1) rotated
//   by the row's angle i: (a, b) -> (a cos - b sin, a sin + b cos);
// bf16 out through the warp's 1 KB shared slab (32 rows x 16 columns), 16
// columns at a time: each lane writes its row's 32 bytes (16-byte halves
// XOR-ed with (row / 4) mod 2: conflict-free), then lane l stores halves l
// and l + 32, i.e. rows l / 2 and 16 + l / 2, as whole 32-byte segments.
// head_bias: the head's 128 bias columns (bf16, shared memory); gamma: the
// part's 128 weights (shared memory); row0: the warp's first row.
SVDQ_DEV void qkv_head(uint32_t (&r)[4][32], const uint16_t* head_bias, const float* gamma, float2 alpha2,
                       const QkvParams& qp, int part, int M, int N, int row, bool row_ok, int row0, int n,
                       uint32_t slab, int lane) {
#pragma unroll
  for (int c4 = 0; c4 < 4; ++c4) {
#pragma unroll
    for (int k8 = 0; k8 < 4; ++k8) {
      const uint4 bw = *reinterpret_cast<const uint4*>(head_bias + 32 * c4 + 8 * k8);
      const uint32_t bb[4] = {bw.x, bw.y, bw.z, bw.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int e = 8 * k8 + 2 * j;
        const float2 v = __ffma2_rn(alpha2, make_float2(__uint_as_float(r[c4][e]), __uint_as_float(r[c4][e + 1])),
                                    bf16x2_to_float2(bb[j]));
        r[c4][e] = __float_as_uint(v.x);
        r[c4][e + 1] = __float_as_uint(v.y);
      }
    }
  }
  if (part < 2) {
    float2 ss = make_float2(0.f, 0.f);
#pragma unroll
    for (int c4 = 0; c4 < 4; ++c4)
#pragma unroll
      for (int e = 0; e < 32; e += 2) {
        const float2 v = make_float2(__uint_as_float(r[c4][e]), __uint_as_float(r[c4][e + 1]));
        ss = __ffma2_rn(v, v, ss);
      }
    const float ms = __fmul_rn(__fadd_rn(ss.x, ss.y), 1.0f / 128.0f);
    const float rn = __frsqrt_rn(__fadd_rn(ms, qp.eps));
    const float2 rn2 = make_float2(rn, rn);
    const float* cs = qp.rope_cos + (row_ok ? row : 0);
    const float* sn = qp.rope_sin + (row_ok ? row : 0);
#pragma unroll
    for (int c4 = 0; c4 < 4; ++c4) {
#pragma unroll
      for (int k4 = 0; k4 < 4; ++k4) {
        // features 32 c4 + 8 k4 .. +7: pairs i = 16 c4 + 4 k4 .. +3
        const float4 g0 = *reinterpret_cast<const float4*>(gamma + 32 * c4 + 8 * k4);
        const float4 g1 = *reinterpret_cast<const float4*>(gamma + 32 * c4 + 8 * k4 + 4);
        const float gg[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const size_t i = (size_t)(16 * c4 + 4 * k4 + j);
          const float cc = __ldg(cs + i * M), sv = __ldg(sn + i * M);
          const int e = 8 * k4 + 2 * j;
          const float2 u =
              __fmul2_rn(__fmul2_rn(make_float2(__uint_as_float(r[c4][e]), __uint_as_float(r[c4][e + 1])), rn2),
                         make_float2(gg[2 * j], gg[2 * j + 1]));
          r[c4][e] = __float_as_uint(__fmaf_rn(u.x, cc, -__fmul_rn(u.y, sv)));
          r[c4][e + 1] = __float_as_uint(__fmaf_rn(u.x, sv, __fmul_rn(u.y, cc)));
        }
      }
    }
  }
#pragma unroll
  for (int c16 = 0; c16 < 8; ++c16) {
    uint32_t w[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = 16 * (c16 & 1) + 2 * j;
      __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(r[c16 >> 1][e]), __uint_as_float(r[c16 >> 1][e + 1]));
      w[j] = *reinterpret_cast<uint32_t*>(&h2);
    }
#pragma unroll
    for (int h = 0; h < 2; ++h)
      st_shared_v4(slab + lane * 32 + ((h ^ ((lane >> 2) & 1)) << 4),
                   make_uint4(w[4 * h], w[4 * h + 1], w[4 * h + 2], w[4 * h + 3]));
    __syncwarp();
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int pc = lane + 32 * k, rr = pc >> 1, h = pc & 1;
      const uint4 v = ld_shared_v4(slab + rr * 32 + ((h ^ ((rr >> 2) & 1)) << 4));
      const int grow = row0 + rr;
      if (grow < M) *reinterpret_cast<uint4*>(qp.y + (size_t)grow * N + n + 16 * c16 + 8 * h) = v;
    }
    __syncwarp();  // the slab's reads precede the next writes
  }
}

}  // namespace svdq
