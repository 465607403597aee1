// S1: smoothing + activation quantization + low-rank down-projection.
//
// Page: "Hugging Face integrates Nunchaku 4-bit diffusion inference into
// Diffusers", section "SVDQuant and the Nunchaku engine": activation outliers
// are migrated into the weights (x_hat = x / lambda per input channel), the
// activations are quantized to 4 bits, and a 16-bit low-rank branch
// x_hat * L1 runs beside them; the engine fuses that down-projection into the
// quantize kernel so the branch costs almost no extra memory traffic.  Here
// the same fusion is one HBM-bound pass over x:
//
//   x_hat = fp32(x) * inv_lambda                       (one fp32 multiply)
//   NVFP4: per 16 along K, a = max|x_hat|, t = a * fp32(1/(6 s_a)), sb = E4M3(t),
//          d = float(sb) * s_a, code = E2M1(x_hat * fp32(1/d))  (RNE, satfinite)
//   INT4:  per 64 along K, sc = bf16(a / 7), q = clamp(rint(x_hat * fp32(1/sc)), -8, 7)
//   u     = x_hat * L1 on tensor cores (mma.sync, fp32 accumulate):
//           NVFP4: x_hat * 2^-e and L1 in fp16 (11-bit significands), with the
//           power of two 2^-e chosen from s_a so that the calibrated range
//           maps to [2^12, 2^13) and nothing overflows; u = acc * 2^e exactly;
//           INT4 (no tensor scale to bound the range): x_hat split into a
//           bf16 hi + lo pair so that u carries ~16 significand bits
//   lora_act[m] = [hi(u * c) | lo(u * c)]  (bf16, 2r values per row), with
//           c = 1 / (s_a s_w) for NVFP4 (folds the GEMM's per-tensor scale)
//           and c = 1 for INT4.
//
// Mapping.  A CTA owns 16 rows; its 16 warps walk interleaved 32-wide K
// blocks.  Lane (g = lane / 4, c = lane % 4) copies 8 consecutive elements of
// rows g and g+8 at k = kb + 8c (16-byte cp.async into its own shared-memory
// ring slots, ahead of the compute); these 16 values are exactly the lane's
// mma.m16n8k16 A fragments for two K=16 steps under the k-permutation
// logical(s, 2c + {0,1}, 2c + 8 + {0,1}) <-> kb + 8c + 4s + {0,1,2,3}; the B
// fragments are loaded with the same permutation from L1^T, so the dot
// products are unchanged.  A 16-group is the lane pair (c, c^1): its amax is
// one shuffle.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

#include "int4_dequant_rows.cuh"
#include "ptx.cuh"
#include "svdq_internal.h"

namespace svdq {

namespace {

constexpr int S1_ROWS = 16;
constexpr int S1_WARPS = 16;
constexpr int S1_THREADS = S1_WARPS * 32;

SVDQ_DEV void unpack8(const uint4& v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

SVDQ_DEV void mma_f16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

SVDQ_DEV uint32_t pack_f16x2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);  // .x = lo (low half)
  return *reinterpret_cast<uint32_t*>(&h);
}

SVDQ_DEV void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Eight fp32 (already multiplied by the block's reciprocal scale) -> eight
// E2M1 codes in one 32-bit word, element 2i in the low nibble of byte i.
SVDQ_DEV uint32_t cvt_e2m1x8(const float (&v)[8], float r) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(out)
      : "f"(__fmul_rn(v[0], r)), "f"(__fmul_rn(v[1], r)), "f"(__fmul_rn(v[2], r)), "f"(__fmul_rn(v[3], r)),
        "f"(__fmul_rn(v[4], r)), "f"(__fmul_rn(v[5], r)), "f"(__fmul_rn(v[6], r)), "f"(__fmul_rn(v[7], r)));
  return out;
}

// x (fp32) -> the bf16 pair words of (hi, lo) with hi = bf16(x), lo = bf16(x - hi),
// for two elements at a time: hi2 / lo2 hold (e0 in the low half, e1 high).
SVDQ_DEV void split_bf16x2(float e0, float e1, uint32_t& hi2, uint32_t& lo2) {
  __nv_bfloat162 h = __floats2bfloat162_rn(e0, e1);
  const uint32_t hb = *reinterpret_cast<uint32_t*>(&h);
  const float h0 = __uint_as_float(hb << 16), h1 = __uint_as_float(hb & 0xFFFF0000u);
  __nv_bfloat162 l = __floats2bfloat162_rn(__fsub_rn(e0, h0), __fsub_rn(e1, h1));
  hi2 = hb;
  lo2 = *reinterpret_cast<uint32_t*>(&l);
}

// Exact E4M3 (non-negative) byte -> fp32 from the format fields.
SVDQ_DEV float e4m3_value(uint32_t b) {
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"((unsigned short)(b & 0xFF)));
  float f;
  asm("cvt.f32.f16 %0, %1;" : "=f"(f) : "h"((unsigned short)(h2 & 0xFFFF)));
  return f;  // E4M3 -> f16 -> f32 are both exact
}

// Byte offset of scale (row, group) in the tiled NVFP4 scale layout:
// 512-byte chunks of 128 rows x 4 groups, chunks ordered (row block, k chunk).
SVDQ_DEV size_t sf_offset(int row, int group, int K) {
  const int kchunks = K / 64;
  return ((size_t)(row >> 7) * kchunks + (group >> 2)) * 512 + (row & 31) * 16 + ((row & 127) >> 5) * 4 + (group & 3);
}

// Per-thread asynchronous prefetch: each lane copies the x and L1^T fragments
// it will consume into its own slots of a shared-memory ring (no other thread
// reads them, so no block-wide synchronisation is needed), PREFETCH units ahead.
SVDQ_DEV void cp_async16(void* smem_dst, const void* gsrc, bool pred) {
  const uint32_t d = smem_u32(smem_dst);
  const int n = pred ? 16 : 0;  // src-size 0 -> the 16 bytes are zero-filled
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(gsrc), "r"(n) : "memory");
}
SVDQ_DEV void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
SVDQ_DEV void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Units whose copies are in flight per warp.  The ring holds PREFETCH x STEP
// slots of 6 x 16 bytes per thread: 96 KB per CTA for NVFP4 with two units,
// 96 KB for INT4 (two 32-blocks per unit) with one.  At two units INT4 would
// take 192 KB, one CTA per SM, and the 256 CTAs of a 4096-row activation two
// waves; with one, two CTAs fit on every SM and the warps of the other CTA
// cover a warp's memory round trip.
template <bool kNvfp4>
constexpr int s1_prefetch() { return kNvfp4 ? 2 : 1; }
// Slot contents per 32-wide block: x rows g and g+8 (2 x 16 B), then the four
// L1^T fragments of the lane (4 x 16 B).
constexpr int S1_SLOT_U4 = 6;

template <bool kNvfp4>
__global__ void __launch_bounds__(S1_THREADS, 2) quantize_act_kernel(QuantActParams p) {
  constexpr int STEP = kNvfp4 ? 1 : 2;  // 32-blocks per unit (INT4 group = 64)
  constexpr int S1_PREFETCH = s1_prefetch<kNvfp4>();
  extern __shared__ uint4 s1_ring[];     // [PREFETCH][STEP][SLOT_U4][THREADS]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const int row0 = blockIdx.x * S1_ROWS + g;
  const int row1 = row0 + 8;
  const bool ok0 = row0 < p.M, ok1 = row1 < p.M;
  const int K = p.K;
  pdl_wait();  // x and the weights of the previous kernel's making
  if constexpr (!kNvfp4) {
    // The blocks past the quantizer's convert the layer's weight rows (they
    // depend on nothing this kernel writes), on the SM slots the quantizer
    // leaves free.
    if (p.w_side.R > 0 && (int)blockIdx.x >= p.s1_blocks) {
      pdl_launch_dependents();
      float* sc = reinterpret_cast<float*>(s1_ring);
      for (int r0 = ((int)blockIdx.x - p.s1_blocks) * 32; r0 < p.w_side.R; r0 += p.w_blocks * 32)
        int4_dequant_rows<32>(p.w_side, r0, sc);
      return;
    }
  }
  const int nunits = K / (32 * STEP);

  const uint16_t* __restrict__ x = p.x;
  const uint16_t* __restrict__ l1t = p.lora_down;  // [r][K]
  const float* __restrict__ inv_lam = p.inv_smooth;

  auto slot = [&](int ring, int h, int q) -> uint4* {
    return s1_ring + (((ring * STEP + h) * S1_SLOT_U4 + q) * S1_THREADS + threadIdx.x);
  };
  // Units of this warp: unit u = warp + S1_WARPS * i.
  const int my_units = nunits > warp ? (nunits - warp + S1_WARPS - 1) / S1_WARPS : 0;
  auto prefetch = [&](int i) {
    if (i < my_units) {
      const int unit = warp + S1_WARPS * i;
      const int ring = i % S1_PREFETCH;
#pragma unroll
      for (int h = 0; h < STEP; ++h) {
        const int k = (unit * STEP + h) * 32 + 8 * c;
        cp_async16(slot(ring, h, 0), x + (size_t)(ok0 ? row0 : 0) * K + k, ok0);
        cp_async16(slot(ring, h, 1), x + (size_t)(ok1 ? row1 : 0) * K + k, ok1);
#pragma unroll
        for (int j = 0; j < 4; ++j) cp_async16(slot(ring, h, 2 + j), l1t + (size_t)(8 * j + g) * K + k, true);
      }
    }
    cp_async_commit();  // always commit (possibly empty) so group counting stays uniform
  };

  float acc[4][4];
#pragma unroll
  for (int j = 0; j < 4; ++j)
#pragma unroll
    for (int q = 0; q < 4; ++q) acc[j][q] = 0.f;

  const float s_a = p.act_scale;
  const float inv_six_s = __frcp_rn(__fmul_rn(6.0f, s_a));

#pragma unroll
  for (int i = 0; i < S1_PREFETCH - 1; ++i) prefetch(i);

  for (int i = 0; i < my_units; ++i) {
    prefetch(i + S1_PREFETCH - 1);
    cp_async_wait<S1_PREFETCH - 1>();
    const int unit = warp + S1_WARPS * i;
    const int ring = i % S1_PREFETCH;
    float v0[STEP][8], v1[STEP][8];  // x_hat for rows g, g+8
#pragma unroll
    for (int h = 0; h < STEP; ++h) {
      const int k = (unit * STEP + h) * 32 + 8 * c;
      const float4 il0 = __ldg(reinterpret_cast<const float4*>(inv_lam + k));
      const float4 il1 = __ldg(reinterpret_cast<const float4*>(inv_lam + k + 4));
      const float il[8] = {il0.x, il0.y, il0.z, il0.w, il1.x, il1.y, il1.z, il1.w};
      unpack8(*slot(ring, h, 0), v0[h]);
      unpack8(*slot(ring, h, 1), v1[h]);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        v0[h][e] = __fmul_rn(v0[h][e], il[e]);
        v1[h][e] = __fmul_rn(v1[h][e], il[e]);
      }
    }

    // ---------------- quantize ----------------
    if constexpr (kNvfp4) {
      float a0 = 0.f, a1 = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        a0 = fmaxf(a0, fabsf(v0[0][e]));
        a1 = fmaxf(a1, fabsf(v1[0][e]));
      }
      a0 = fmaxf(a0, __shfl_xor_sync(0xffffffffu, a0, 1));
      a1 = fmaxf(a1, __shfl_xor_sync(0xffffffffu, a1, 1));
      // The two lanes of a pair share both groups: the even lane derives row
      // g's scale, the odd lane row g+8's, and they swap the results.
      const bool odd = (c & 1) != 0;
      const uint32_t sb_m = cvt_e4m3(__fmul_rn(odd ? a1 : a0, inv_six_s));
      const float d_m = __fmul_rn(e4m3_value(sb_m), s_a);
      const float r_m = d_m != 0.f ? __frcp_rn(d_m) : 0.f;  // 0 marks an all-zero group
      const float r_o = __shfl_xor_sync(0xffffffffu, r_m, 1);
      const uint32_t sb_o = __shfl_xor_sync(0xffffffffu, sb_m, 1);
      const float r0 = odd ? r_o : r_m, r1 = odd ? r_m : r_o;
      const uint32_t sb0 = odd ? sb_o : sb_m, sb1 = odd ? sb_m : sb_o;
      const uint32_t w0 = r0 != 0.f ? cvt_e2m1x8(v0[0], r0) : 0u;
      const uint32_t w1 = r1 != 0.f ? cvt_e2m1x8(v1[0], r1) : 0u;
      const int k = unit * 32 + 8 * c;
      uint8_t* codes = p.act_codes;
      if (ok0) __stcs(reinterpret_cast<unsigned int*>(codes + (size_t)row0 * (K / 2) + k / 2), w0);
      if (ok1) __stcs(reinterpret_cast<unsigned int*>(codes + (size_t)row1 * (K / 2) + k / 2), w1);
      if ((c & 1) == 0) {
        const int grp = k >> 4;
        p.act_scales[sf_offset(row0, grp, K)] = (uint8_t)sb0;  // rows >= M get 0 (zero input)
        p.act_scales[sf_offset(row1, grp, K)] = (uint8_t)sb1;
      }
    } else {
      // INT4: group of 64 = lanes c=0..3 over two 32-blocks.
      float a0 = 0.f, a1 = 0.f;
#pragma unroll
      for (int h = 0; h < STEP; ++h)
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          a0 = fmaxf(a0, fabsf(v0[h][e]));
          a1 = fmaxf(a1, fabsf(v1[h][e]));
        }
      a0 = fmaxf(a0, __shfl_xor_sync(0xffffffffu, a0, 1));
      a1 = fmaxf(a1, __shfl_xor_sync(0xffffffffu, a1, 1));
      a0 = fmaxf(a0, __shfl_xor_sync(0xffffffffu, a0, 2));
      a1 = fmaxf(a1, __shfl_xor_sync(0xffffffffu, a1, 2));
      const __nv_bfloat16 sc0 = __float2bfloat16_rn(__fdiv_rn(a0, 7.0f));
      const __nv_bfloat16 sc1 = __float2bfloat16_rn(__fdiv_rn(a1, 7.0f));
      const float f0 = __bfloat162float(sc0), f1 = __bfloat162float(sc1);
      const float r0 = __frcp_rn(f0), r1 = __frcp_rn(f1);
#pragma unroll
      for (int h = 0; h < STEP; ++h) {
        uint32_t w0 = 0, w1 = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          int q0 = 0, q1 = 0;
          if (f0 != 0.f) q0 = max(-8, min(7, __float2int_rn(__fmul_rn(v0[h][e], r0))));
          if (f1 != 0.f) q1 = max(-8, min(7, __float2int_rn(__fmul_rn(v1[h][e], r1))));
          w0 |= (uint32_t)(q0 & 0xF) << (4 * e);
          w1 |= (uint32_t)(q1 & 0xF) << (4 * e);
        }
        const int k = (unit * STEP + h) * 32 + 8 * c;
        if (ok0) __stcs(reinterpret_cast<unsigned int*>(p.act_codes + (size_t)row0 * (K / 2) + k / 2), w0);
        if (ok1) __stcs(reinterpret_cast<unsigned int*>(p.act_codes + (size_t)row1 * (K / 2) + k / 2), w1);
      }
      if (c == 0) {
        // INT4 activation scales: bf16, group-major [K/64][M_pad].
        uint16_t* sc = reinterpret_cast<uint16_t*>(p.act_scales);
        sc[(size_t)unit * p.M_pad + row0] = __bfloat16_as_ushort(sc0);
        sc[(size_t)unit * p.M_pad + row1] = __bfloat16_as_ushort(sc1);
      }
    }

    // ---------------- low-rank down-projection ----------------
    if constexpr (kNvfp4) {
      const float xs = p.lr_in_scale;
      uint32_t a[2][4];
#pragma unroll
      for (int st = 0; st < 2; ++st) {
        // A fragment registers: (row g, k 0-1), (row g+8, k 0-1), (row g, k 2-3), (row g+8, k 2-3)
        a[st][0] = pack_f16x2(__fmul_rn(v0[0][4 * st + 0], xs), __fmul_rn(v0[0][4 * st + 1], xs));
        a[st][1] = pack_f16x2(__fmul_rn(v1[0][4 * st + 0], xs), __fmul_rn(v1[0][4 * st + 1], xs));
        a[st][2] = pack_f16x2(__fmul_rn(v0[0][4 * st + 2], xs), __fmul_rn(v0[0][4 * st + 3], xs));
        a[st][3] = pack_f16x2(__fmul_rn(v1[0][4 * st + 2], xs), __fmul_rn(v1[0][4 * st + 3], xs));
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint4 bw = *slot(ring, 0, 2 + j);
        mma_f16_16816(acc[j], a[0], bw.x, bw.y);
        mma_f16_16816(acc[j], a[1], bw.z, bw.w);
      }
    } else {
#pragma unroll
    for (int h = 0; h < STEP; ++h) {
      uint32_t ahi[2][4], alo[2][4];
#pragma unroll
      for (int st = 0; st < 2; ++st) {
        // A fragment registers: (row g, k 0-1), (row g+8, k 0-1), (row g, k 2-3), (row g+8, k 2-3)
        split_bf16x2(v0[h][4 * st + 0], v0[h][4 * st + 1], ahi[st][0], alo[st][0]);
        split_bf16x2(v1[h][4 * st + 0], v1[h][4 * st + 1], ahi[st][1], alo[st][1]);
        split_bf16x2(v0[h][4 * st + 2], v0[h][4 * st + 3], ahi[st][2], alo[st][2]);
        split_bf16x2(v1[h][4 * st + 2], v1[h][4 * st + 3], ahi[st][3], alo[st][3]);
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint4 bw = *slot(ring, h, 2 + j);
        mma_bf16_16816(acc[j], ahi[0], bw.x, bw.y);
        mma_bf16_16816(acc[j], alo[0], bw.x, bw.y);
        mma_bf16_16816(acc[j], ahi[1], bw.z, bw.w);
        mma_bf16_16816(acc[j], alo[1], bw.z, bw.w);
      }
    }
    }
  }
  cp_async_wait<0>();

  // Let the GEMM that consumes these outputs start its prologue.
  pdl_launch_dependents();

  // ---------------- cross-warp reduction of u, then the bf16 hi/lo fold ----
  // (reuses the prefetch ring: every copy has landed and been consumed)
  __syncthreads();
  float(*red)[S1_ROWS][33] = reinterpret_cast<float(*)[S1_ROWS][33]>(s1_ring);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    red[warp][g][8 * j + 2 * c] = acc[j][0];
    red[warp][g][8 * j + 2 * c + 1] = acc[j][1];
    red[warp][g + 8][8 * j + 2 * c] = acc[j][2];
    red[warp][g + 8][8 * j + 2 * c + 1] = acc[j][3];
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < S1_ROWS * 32; idx += S1_THREADS) {
    const int r = idx >> 5, col = idx & 31;
    float u = 0.f;
#pragma unroll
    for (int w = 0; w < S1_WARPS; ++w) u = __fadd_rn(u, red[w][r][col]);
    const int row = blockIdx.x * S1_ROWS + r;
    if (row < p.M) {
      const float uf = __fmul_rn(u, p.lora_scale);  // lora_scale also undoes 2^-e (NVFP4)
      const __nv_bfloat16 hi = __float2bfloat16_rn(uf);
      const __nv_bfloat16 lo = __float2bfloat16_rn(__fsub_rn(uf, __bfloat162float(hi)));
      uint16_t* la = p.lora_act + (size_t)row * 64;
      la[col] = __bfloat16_as_ushort(hi);
      la[32 + col] = __bfloat16_as_ushort(lo);
    }
  }
}

}  // namespace

bool int4_weight_side_fits(int K) {
  return int4_dequant_rows_smem(32, K) <= (size_t)s1_prefetch<false>() * 2 * S1_SLOT_U4 * S1_THREADS * sizeof(uint4);
}

cudaError_t launch_quantize_act(const QuantActParams& p, bool nvfp4, cudaStream_t stream, bool pdl) {
  if (!nvfp4 && p.w_side.R > 0 && !int4_weight_side_fits(p.K)) return cudaErrorInvalidValue;
  const int rows_pad = p.M_pad;  // cover scale padding rows too (they get zero scales)
  dim3 grid((rows_pad + S1_ROWS - 1) / S1_ROWS + (!nvfp4 && p.w_side.R > 0 ? p.w_blocks : 0));
  const size_t ring_bytes = (size_t)(nvfp4 ? s1_prefetch<true>() : s1_prefetch<false>()) * (nvfp4 ? 1 : 2) *
                            S1_SLOT_U4 * S1_THREADS * sizeof(uint4);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(S1_THREADS);
  cfg.dynamicSmemBytes = ring_bytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  set_pdl(cfg, attr, pdl);
  cudaError_t e;
  if (nvfp4) {
    e = cudaFuncSetAttribute(quantize_act_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ring_bytes);
    if (e != cudaSuccess) return e;
    return cudaLaunchKernelEx(&cfg, quantize_act_kernel<true>, p);
  }
  e = cudaFuncSetAttribute(quantize_act_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ring_bytes);
  if (e != cudaSuccess) return e;
  return cudaLaunchKernelEx(&cfg, quantize_act_kernel<false>, p);
}

}  // namespace svdq
