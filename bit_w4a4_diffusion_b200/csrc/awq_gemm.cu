// S4: AWQ W4A16 linear, y = bf16(x deq(W)^T + b), deq = (q - z) * sc per 64.
//
// Pages: "Nunchaku Lite" docs, "Supported quantization types" table
// (awq_w4a16, int4, group 64); "Hugging Face integrates Nunchaku 4-bit
// diffusion inference into Diffusers", list of kernel families (memory-bound,
// precision-sensitive modulation layers such as adaptive-norm projections).
//
// For M <= 16 tokens the layer is a weight stream: 0.5 byte per weight plus
// group metadata.  The kernel reads every weight byte once with coalesced
// loads and does the arithmetic on tensor cores with the weight as the
// 16-row operand:  D[n, m] = sum_k (q - z)[n, k] * x[m, k]  per 64-group
// (exact: |q - z| <= 15 is exact in bf16 and each product is exact in fp32),
// then acc[n, m] += sc[n, g] * D[n, m] in fp32.
//
// Mapping: a CTA owns 16 weight rows; its 4 warps split K.  Lane
// (g = lane/4, c = lane%4) holds 16 codes (8 bytes) of rows g and g+8 at
// k = 64G + 16c within group G.  Four m16n8k16 steps cover the group; step s
// uses physical k = 64G + 16c + 4s + {0,1,2,3} for the lane's logical k pairs
// (2c, 2c+1) and (2c+8, 2c+9); x is loaded with the same permutation.
// (q - z) is formed with the magic-number trick: bf16 bits 0x4300|q encode
// 128 + q exactly, and subtracting 128 + z leaves q - z.
#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"
#include "svdq_internal.h"

namespace svdq {
namespace {

constexpr int AWQ_ROWS = 16;
constexpr int AWQ_WARPS = 4;
constexpr int AWQ_UNROLL = 4;  // groups whose loads are issued together

SVDQ_DEV void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Byte j of `lo_nib` / `hi_nib` (the low / high nibbles of four code bytes)
// -> bf16x2 {128 + lo, 128 + hi} - {128 + z, 128 + z} = {lo - z, hi - z}.
SVDQ_DEV uint32_t dequant_pair(uint32_t lo_nib, uint32_t hi_nib, int j, uint32_t zz) {
  // Selector nibble n picks result byte n: byte 0 <- lo_j, byte 2 <- hi_j.
  const uint32_t sel = (uint32_t)j | ((uint32_t)(4 + j) << 8);
  uint32_t v = __byte_perm(lo_nib, hi_nib, sel);
  v = (v & 0x00FF00FFu) | 0x43004300u;
  __nv_bfloat162 r = __hsub2(*reinterpret_cast<__nv_bfloat162*>(&v), *reinterpret_cast<const __nv_bfloat162*>(&zz));
  return *reinterpret_cast<uint32_t*>(&r);
}

template <int MT>
__global__ void __launch_bounds__(AWQ_WARPS * 32) awq_kernel(AwqParams p) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const int n0 = blockIdx.x * AWQ_ROWS;
  const int rA = n0 + g, rB = n0 + g + 8;
  const int K = p.K;
  pdl_wait();  // x of the previous kernel's making
  const int ngroups = K / 64;
  const int gpw = (ngroups + AWQ_WARPS - 1) / AWQ_WARPS;  // groups per warp
  const int G_begin = warp * gpw;
  const int G_end = min(ngroups, G_begin + gpw);

  float acc[MT][4];
#pragma unroll
  for (int t = 0; t < MT; ++t)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[t][i] = 0.f;

  const uint8_t* __restrict__ qw = p.qweight;
  const uint16_t* __restrict__ x = p.x;

  for (int G0 = G_begin; G0 < G_end; G0 += AWQ_UNROLL) {
    uint2 wa[AWQ_UNROLL], wb[AWQ_UNROLL];
    float sa[AWQ_UNROLL], sb[AWQ_UNROLL];
    uint32_t za[AWQ_UNROLL], zb[AWQ_UNROLL];
#pragma unroll
    for (int u = 0; u < AWQ_UNROLL; ++u) {
      const int G = G0 + u;
      if (G < G_end) {
        const size_t off = (size_t)(64 * G + 16 * c) / 2;
        wa[u] = __ldg(reinterpret_cast<const uint2*>(qw + (size_t)rA * (K / 2) + off));
        wb[u] = __ldg(reinterpret_cast<const uint2*>(qw + (size_t)rB * (K / 2) + off));
        sa[u] = __bfloat162float(__ushort_as_bfloat16(__ldg(p.scales + (size_t)rA * ngroups + G)));
        sb[u] = __bfloat162float(__ushort_as_bfloat16(__ldg(p.scales + (size_t)rB * ngroups + G)));
        za[u] = (__ldg(p.zeros + (size_t)rA * (K / 128) + G / 2) >> (4 * (G & 1))) & 0xF;
        zb[u] = (__ldg(p.zeros + (size_t)rB * (K / 128) + G / 2) >> (4 * (G & 1))) & 0xF;
      }
    }
#pragma unroll
    for (int u = 0; u < AWQ_UNROLL; ++u) {
      const int G = G0 + u;
      if (G >= G_end) break;
      const uint32_t zza = (0x4300u | za[u]) * 0x10001u;
      const uint32_t zzb = (0x4300u | zb[u]) * 0x10001u;
      const uint32_t wA[2] = {wa[u].x, wa[u].y}, wB[2] = {wb[u].x, wb[u].y};
      float part[MT][4];
#pragma unroll
      for (int t = 0; t < MT; ++t)
#pragma unroll
        for (int i = 0; i < 4; ++i) part[t][i] = 0.f;
      // x fragments for this lane: rows m = 8t + g, k = 64G + 16c + [0, 16)
      uint4 xv[MT][2];
#pragma unroll
      for (int t = 0; t < MT; ++t) {
        const int m = 8 * t + g;
        if (m < p.M) {
          const uint4* xp = reinterpret_cast<const uint4*>(x + (size_t)m * K + 64 * G + 16 * c);
          xv[t][0] = __ldg(xp);
          xv[t][1] = __ldg(xp + 1);
        } else {
          xv[t][0] = make_uint4(0, 0, 0, 0);
          xv[t][1] = make_uint4(0, 0, 0, 0);
        }
      }
#pragma unroll
      for (int h = 0; h < 2; ++h) {  // word h holds steps 2h, 2h+1
        const uint32_t loA = wA[h] & 0x0F0F0F0Fu, hiA = (wA[h] >> 4) & 0x0F0F0F0Fu;
        const uint32_t loB = wB[h] & 0x0F0F0F0Fu, hiB = (wB[h] >> 4) & 0x0F0F0F0Fu;
#pragma unroll
        for (int ss = 0; ss < 2; ++ss) {
          const int s = 2 * h + ss;
          uint32_t a[4];
          a[0] = dequant_pair(loA, hiA, 2 * ss, zza);      // row g,   k-pair (0,1)
          a[1] = dequant_pair(loB, hiB, 2 * ss, zzb);      // row g+8
          a[2] = dequant_pair(loA, hiA, 2 * ss + 1, zza);  // row g,   k-pair (2,3)
          a[3] = dequant_pair(loB, hiB, 2 * ss + 1, zzb);  // row g+8
#pragma unroll
          for (int t = 0; t < MT; ++t) {
            const uint4& xq = xv[t][s >> 1];
            const uint32_t b0 = (s & 1) ? xq.z : xq.x;
            const uint32_t b1 = (s & 1) ? xq.w : xq.y;
            mma16816(part[t], a, b0, b1);
          }
        }
      }
#pragma unroll
      for (int t = 0; t < MT; ++t) {
        acc[t][0] = __fmaf_rn(sa[u], part[t][0], acc[t][0]);
        acc[t][1] = __fmaf_rn(sa[u], part[t][1], acc[t][1]);
        acc[t][2] = __fmaf_rn(sb[u], part[t][2], acc[t][2]);
        acc[t][3] = __fmaf_rn(sb[u], part[t][3], acc[t][3]);
      }
    }
  }

  // D fragment: (row g | g+8, col m = 8t + 2c + {0,1}).  Reduce over warps.
  __shared__ float red[AWQ_WARPS][AWQ_ROWS][16 + 1];
#pragma unroll
  for (int t = 0; t < MT; ++t) {
    red[warp][g][8 * t + 2 * c] = acc[t][0];
    red[warp][g][8 * t + 2 * c + 1] = acc[t][1];
    red[warp][g + 8][8 * t + 2 * c] = acc[t][2];
    red[warp][g + 8][8 * t + 2 * c + 1] = acc[t][3];
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < AWQ_ROWS * 8 * MT; idx += AWQ_WARPS * 32) {
    const int m = idx / AWQ_ROWS, r = idx % AWQ_ROWS;
    if (m >= p.M) continue;
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < AWQ_WARPS; ++w) v = __fadd_rn(v, red[w][r][m]);
    const int n = n0 + r;
    if (p.bias) v = __fadd_rn(v, __bfloat162float(__ushort_as_bfloat16(p.bias[n])));
    p.y[(size_t)m * p.N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
  }
}

}  // namespace

cudaError_t launch_awq(const AwqParams& p, int num_sms, cudaStream_t stream, bool pdl) {
  (void)num_sms;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.N / AWQ_ROWS);
  cfg.blockDim = dim3(AWQ_WARPS * 32);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  set_pdl(cfg, attr, pdl);
  if (p.M <= 8) return cudaLaunchKernelEx(&cfg, awq_kernel<1>, p);
  return cudaLaunchKernelEx(&cfg, awq_kernel<2>, p);
}

}  // namespace svdq
