// S1 for NVFP4, TMA-fed: smoothing + activation quantization + low-rank
// down-projection in one pass over x.
//
// Page: "Hugging Face integrates Nunchaku 4-bit diffusion inference into
// Diffusers", section "SVDQuant and the Nunchaku engine": outliers migrate
// into the weights (x_hat = x / lambda per input channel), the activations are
// quantized to 4 bits and a 16-bit low-rank branch x_hat * L1 runs beside
// them, fused into the quantize kernel.  Arithmetic (that of the
// per-thread-copy kernel in quantize_act.cu: the same codes and scales bit
// for bit, u summed over K in a different order):
//
//   x_hat = fp32(x) * inv_lambda
//   per 16 along K: a = max|x_hat|, sb = E4M3(a * fp32(1/(6 s_a))),
//     d = float(sb) * s_a, code = E2M1(x_hat * fp32(1/d))     (RNE, satfinite)
//   u = (x_hat * 2^-e in fp16) . (L1 in fp16) on tensor cores, fp32 accumulate
//   lora_act[m] = [hi(u c) | lo(u c)],  c = 2^e / (s_a s_w)
//
// Why a second kernel: with 16 rows per CTA and per-thread cp.async
// prefetch one 32-wide block ahead, each warp of the first kernel walks only
// a few blocks, each a full memory round trip, and every CTA pulls all of
// L1^T (twice the bytes of its x rows) from L2.  Here a CTA owns 32 rows (so
// L1^T is read once per 32 rows), one producer warp streams 256-wide K slices
// of x, L1^T and 1/lambda into a six-stage shared-memory ring with TMA, and 16
// compute warps consume them: warp w takes the 32-wide block (w mod 8) of
// every slice for rows [16 (w / 8), 16 (w / 8) + 16).  Lane (g, c) holds 8
// consecutive elements of two rows, which are its mma.m16n8k16 A fragments
// under the k-permutation of the first kernel.
//
// Two orderings keep the memory system busy.  CTA b walks the K slices
// starting at slice b mod (K / 256): in lockstep every CTA would read the
// same 16 KB of L1^T from the same few L2 slices at once.  And lane (g, c)
// takes rows (and ranks) perm(g), perm(g) + 8 with perm = 0 4 1 5 2 6 3 7:
// the 128-byte swizzle places rows r and r + 1 in the same bank groups, so
// the two rows of one quarter-warp load must differ in bit 2 to avoid a
// two-way bank conflict.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

#include "ptx.cuh"
#include "svdq_internal.h"

namespace svdq {
namespace {

constexpr int QN_ROWS = 32;                       // rows per CTA
constexpr int QN_SLICE = 256;                     // K elements per stage
constexpr int QN_STAGES = 6;
constexpr int QN_COMPUTE_WARPS = 16;
constexpr int QN_THREADS = (QN_COMPUTE_WARPS + 1) * 32;   // + the producer warp
constexpr int QN_BOX_BYTES = QN_ROWS * 128;               // one 64-wide SWIZZLE_128B box, 32 rows
constexpr int QN_X_BYTES = 4 * QN_BOX_BYTES;              // 16 KB
constexpr int QN_L_BYTES = 4 * QN_BOX_BYTES;              // L1^T, 32 ranks: 16 KB
constexpr int QN_I_BYTES = QN_SLICE * 4;                  // 1/lambda: 1 KB
constexpr int QN_STAGE_BYTES = QN_X_BYTES + QN_L_BYTES + QN_I_BYTES;
static_assert(QN_STAGE_BYTES % 1024 == 0, "stages keep the 1024-byte alignment of SWIZZLE_128B");
// Cross-warp reduction of u: 8 block-warps x 32 rows x 33 (padded) fp32.
constexpr int QN_RED_BYTES = 8 * QN_ROWS * 33 * 4;
static_assert(QN_RED_BYTES <= QN_STAGES * QN_STAGE_BYTES, "the reduction reuses the ring");

struct QnCtl {
  uint64_t full[QN_STAGES];
  uint64_t empty[QN_STAGES];
  int abort_flag;
};

// 1/d for every E4M3 scale byte (d = E4M3(b) * s_a), 0 where d = 0.
constexpr int QN_RCP_BYTES = 256 * 4;
constexpr size_t QN_SMEM_BYTES = 1024 + QN_STAGES * QN_STAGE_BYTES + QN_RCP_BYTES + sizeof(QnCtl);
constexpr unsigned long long kQnDrainLimitNs = 2000000000ull;

// Address of the 16-byte chunk holding elements [8 j, 8 j + 8) of row r in a
// 64-wide SWIZZLE_128B box (128-byte rows, 16-byte chunks XOR-ed by r mod 8).
SVDQ_DEV uint32_t sw128_chunk(uint32_t box, int r, int j) {
  return box + (uint32_t)r * 128u + (uint32_t)((j ^ (r & 7)) << 4);
}

SVDQ_DEV uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

SVDQ_DEV void mma_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

SVDQ_DEV uint32_t f16x2(float lo, float hi) {
  uint32_t out;
  asm("cvt.rn.f16x2.f32 %0, %2, %1;" : "=r"(out) : "f"(lo), "f"(hi));
  return out;  // lo in the low half
}

// Eight fp32 (pairs lo, hi) -> four bytes of E2M1 codes, element 2i in bits
// 8i..8i+3 and element 2i+1 in bits 8i+4..8i+7; RNE, satfinite.
SVDQ_DEV uint32_t e2m1x8(float2 a, float2 b, float2 c, float2 d) {
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

// Exact E4M3 (non-negative) byte -> fp32.
SVDQ_DEV float e4m3_to_float(uint32_t b) {
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"((unsigned short)(b & 0xFF)));
  return __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFF)));
}

SVDQ_DEV size_t scale_offset(int row, int group, int K) {
  const int kchunks = K / 64;
  return ((size_t)(row >> 7) * kchunks + (group >> 2)) * 512 + (row & 31) * 16 + ((row & 127) >> 5) * 4 + (group & 3);
}

__global__ void __launch_bounds__(QN_THREADS, 1)
    quantize_nvfp4_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_l1t,
                          const QuantActParams p, int* dev_status, unsigned long long timeout_ns) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* rcp_tab = reinterpret_cast<float*>(smem + QN_STAGES * QN_STAGE_BYTES);
  QnCtl* ctl = reinterpret_cast<QnCtl*>(smem + QN_STAGES * QN_STAGE_BYTES + QN_RCP_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int K = p.K;
  const int nslices = K / QN_SLICE;
  const int row_base = blockIdx.x * QN_ROWS;
  const int slice0 = (int)(blockIdx.x % (unsigned)nslices);   // this CTA's first K slice
  pdl_wait();  // x of the previous kernel's making

  if (threadIdx.x < 256) {
    // The reciprocal each group's codes are scaled by, for every scale byte
    // the quantizer can produce (the formula of the per-group computation).
    const float d = __fmul_rn(e4m3_to_float(threadIdx.x), p.act_scale);
    rcp_tab[threadIdx.x] = d != 0.f ? __frcp_rn(d) : 0.f;   // 0 marks an all-zero group
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < QN_STAGES; ++s) {
      mbar_init(smem_u32(&ctl->full[s]), 1);
      mbar_init(smem_u32(&ctl->empty[s]), QN_COMPUTE_WARPS);
    }
    ctl->abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  WaitCtx wctx{&ctl->abort_flag, dev_status, timeout_ns};

  if (warp == QN_COMPUTE_WARPS) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tmap(&tm_x);
      prefetch_tmap(&tm_l1t);
      uint32_t issued_mask = 0, issued_phase = 0;
      for (int sl = 0; sl < nslices; ++sl) {
        const int stage = sl % QN_STAGES;
        const uint32_t phase = (uint32_t)(sl / QN_STAGES) & 1;
        if (!mbar_wait(smem_u32(&ctl->empty[stage]), phase ^ 1, wctx, kDevTimeoutProducer)) break;
        const uint32_t base = smem_u32(smem + stage * QN_STAGE_BYTES);
        const uint32_t full = smem_u32(&ctl->full[stage]);
        const int ks = sl + slice0 < nslices ? sl + slice0 : sl + slice0 - nslices;
        const int k0 = ks * QN_SLICE;
        mbar_arrive_expect_tx(full, QN_STAGE_BYTES);
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          tma_load_2d(base + b * QN_BOX_BYTES, &tm_x, k0 + 64 * b, row_base, full);
          tma_load_2d(base + QN_X_BYTES + b * QN_BOX_BYTES, &tm_l1t, k0 + 64 * b, 0, full);
        }
        bulk_load(base + QN_X_BYTES + QN_L_BYTES, p.inv_smooth + k0, QN_I_BYTES, full);
        issued_mask |= 1u << stage;
        issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
      }
      // Never leave with copies in flight into shared memory.
      volatile int never = 0;
      WaitCtx drain_ctx{&never, dev_status, kQnDrainLimitNs};
      for (int s = 0; s < QN_STAGES; ++s)
        if (issued_mask & (1u << s))
          mbar_wait(smem_u32(&ctl->full[s]), (issued_phase >> s) & 1, drain_ctx, kDevTimeoutDrain);
    }
  } else {
    // ------------------------------------------------------------ compute warps
    const int blk = warp & 7;            // 32-wide block within each slice
    const int half = warp >> 3;          // rows [16 half, 16 half + 16)
    const int g = lane >> 2, c = lane & 3;
    const int pg = ((g & 1) << 2) | (g >> 1);            // perm(g): see the header
    const int r0 = 16 * half + pg, r1 = r0 + 8;          // rows within the CTA
    const int row0 = row_base + r0, row1 = row_base + r1;
    const bool ok0 = row0 < p.M, ok1 = row1 < p.M;
    const int box = blk >> 1;                            // 64-wide box holding this block
    const int chunk = (blk & 1) * 4 + c;                 // 16-byte chunk of the lane in that box
    const float s_a = p.act_scale;
    const float inv_six_s = __frcp_rn(__fmul_rn(6.0f, s_a));
    const float2 xs2 = make_float2(p.lr_in_scale, p.lr_in_scale);
    const bool odd = (c & 1) != 0;
    float acc[4][4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[j][q] = 0.f;
    // This lane's code word and (even lanes) scale byte of K slice 0; slice
    // ks adds ks * 128 code bytes and ks * 2048 scale bytes (the tiled scale
    // layout: group 16 ks + 2 blk + c / 2).
    uint8_t* const code0 = p.act_codes + (size_t)row0 * (K / 2) + blk * 16 + 4 * c;
    uint8_t* const code1 = p.act_codes + (size_t)row1 * (K / 2) + blk * 16 + 4 * c;
    uint8_t* const sc0 = p.act_scales + scale_offset(row0, 2 * blk + (c >> 1), K);
    uint8_t* const sc1 = p.act_scales + scale_offset(row1, 2 * blk + (c >> 1), K);

    for (int sl = 0; sl < nslices; ++sl) {
      const int stage = sl % QN_STAGES;
      const uint32_t phase = (uint32_t)(sl / QN_STAGES) & 1;
      const bool got = mbar_wait(smem_u32(&ctl->full[stage]), phase, wctx, kDevTimeoutEpilogue);
      if (!__all_sync(0xffffffffu, got)) break;  // warp-uniform
      const uint32_t base = smem_u32(smem + stage * QN_STAGE_BYTES);
      const uint32_t xbox = base + box * QN_BOX_BYTES;
      const uint32_t lbox = base + QN_X_BYTES + box * QN_BOX_BYTES;
      const uint4 xa = lds128(sw128_chunk(xbox, r0, chunk));
      const uint4 xb = lds128(sw128_chunk(xbox, r1, chunk));
      const uint32_t iaddr = base + QN_X_BYTES + QN_L_BYTES + (uint32_t)(blk * 32 + 8 * c) * 4;
      const uint4 i0 = lds128(iaddr), i1 = lds128(iaddr + 16);
      uint4 bw[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) bw[j] = lds128(sw128_chunk(lbox, 8 * j + pg, chunk));   // rank 8 j + perm(g)
      // Every read of this stage is in registers: release it.
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&ctl->empty[stage]));

      // x_hat for rows g and g+8: bf16 -> fp32, times 1/lambda (two at a time).
      const uint32_t wa[4] = {xa.x, xa.y, xa.z, xa.w}, wb[4] = {xb.x, xb.y, xb.z, xb.w};
      const float il[8] = {__uint_as_float(i0.x), __uint_as_float(i0.y), __uint_as_float(i0.z),
                           __uint_as_float(i0.w), __uint_as_float(i1.x), __uint_as_float(i1.y),
                           __uint_as_float(i1.z), __uint_as_float(i1.w)};
      float2 v0[4], v1[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 ilp = make_float2(il[2 * i], il[2 * i + 1]);
        v0[i] = __fmul2_rn(make_float2(__uint_as_float(wa[i] << 16), __uint_as_float(wa[i] & 0xFFFF0000u)), ilp);
        v1[i] = __fmul2_rn(make_float2(__uint_as_float(wb[i] << 16), __uint_as_float(wb[i] & 0xFFFF0000u)), ilp);
      }

      // ---- NVFP4 quantization: the group of 16 is the lane pair (c, c^1).
      float a0 = 0.f, a1 = 0.f;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a0 = fmaxf(a0, fmaxf(fabsf(v0[i].x), fabsf(v0[i].y)));
        a1 = fmaxf(a1, fmaxf(fabsf(v1[i].x), fabsf(v1[i].y)));
      }
      a0 = fmaxf(a0, __shfl_xor_sync(0xffffffffu, a0, 1));
      a1 = fmaxf(a1, __shfl_xor_sync(0xffffffffu, a1, 1));
      // The even lane derives row g's scale, the odd lane row g+8's; they swap.
      const uint32_t sb_m = cvt_e4m3(__fmul_rn(odd ? a1 : a0, inv_six_s));
      const float r_m = rcp_tab[sb_m & 0xFF];                   // 0 marks an all-zero group
      const float r_o = __shfl_xor_sync(0xffffffffu, r_m, 1);
      const uint32_t sb_o = __shfl_xor_sync(0xffffffffu, sb_m, 1);
      const float q0 = odd ? r_o : r_m, q1 = odd ? r_m : r_o;
      // An all-zero group (scale byte 0) gets all-zero codes, also where a
      // value is -0 or a tiny negative.
      const float2 qq0 = make_float2(q0, q0), qq1 = make_float2(q1, q1);
      const uint32_t w0 = q0 != 0.f ? e2m1x8(__fmul2_rn(v0[0], qq0), __fmul2_rn(v0[1], qq0), __fmul2_rn(v0[2], qq0),
                                             __fmul2_rn(v0[3], qq0))
                                    : 0u;
      const uint32_t w1 = q1 != 0.f ? e2m1x8(__fmul2_rn(v1[0], qq1), __fmul2_rn(v1[1], qq1), __fmul2_rn(v1[2], qq1),
                                             __fmul2_rn(v1[3], qq1))
                                    : 0u;
      const int ks = sl + slice0 < nslices ? sl + slice0 : sl + slice0 - nslices;
      if (ok0) __stcs(reinterpret_cast<unsigned int*>(code0 + ks * (QN_SLICE / 2)), w0);
      if (ok1) __stcs(reinterpret_cast<unsigned int*>(code1 + ks * (QN_SLICE / 2)), w1);
      if (!odd) {
        // 16 groups of 16 per slice = 4 chunks of 512 scale bytes.
        sc0[(size_t)ks * 2048] = (uint8_t)sb_m;  // rows >= M: zero input, scale 0
        sc1[(size_t)ks * 2048] = (uint8_t)sb_o;
      }

      // ---- low-rank down-projection: A = x_hat * 2^-e in fp16.
      uint32_t a[2][4];
#pragma unroll
      for (int st = 0; st < 2; ++st) {
        const float2 p00 = __fmul2_rn(v0[2 * st], xs2), p01 = __fmul2_rn(v0[2 * st + 1], xs2);
        const float2 p10 = __fmul2_rn(v1[2 * st], xs2), p11 = __fmul2_rn(v1[2 * st + 1], xs2);
        // (row g, k 0-1), (row g+8, k 0-1), (row g, k 2-3), (row g+8, k 2-3) of k-step st
        a[st][0] = f16x2(p00.x, p00.y);
        a[st][1] = f16x2(p10.x, p10.y);
        a[st][2] = f16x2(p01.x, p01.y);
        a[st][3] = f16x2(p11.x, p11.y);
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        mma_f16(acc[j], a[0], bw[j].x, bw[j].y);
        mma_f16(acc[j], a[1], bw[j].z, bw[j].w);
      }
    }

    // Let the GEMM that consumes these outputs start its prologue.
    pdl_launch_dependents();

    // ---- cross-warp reduction of u over the 8 block-warps of each half.
    // Every stage was released by all compute warps only after its reads, and
    // the producer waits for each of its loads before leaving, so the ring is
    // free once all threads pass this barrier.
    __syncwarp();
    asm volatile("bar.sync 1, %0;" ::"n"(QN_COMPUTE_WARPS * 32));
    float(*red)[QN_ROWS][33] = reinterpret_cast<float(*)[QN_ROWS][33]>(smem);
    // Accumulator columns 2c, 2c + 1 of n-tile j are ranks 8 j + perm(2c) =
    // 8 j + c and 8 j + perm(2c + 1) = 8 j + 4 + c.
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      red[blk][r0][8 * j + c] = acc[j][0];
      red[blk][r0][8 * j + 4 + c] = acc[j][1];
      red[blk][r1][8 * j + c] = acc[j][2];
      red[blk][r1][8 * j + 4 + c] = acc[j][3];
    }
    asm volatile("bar.sync 1, %0;" ::"n"(QN_COMPUTE_WARPS * 32));
    for (int idx = threadIdx.x; idx < QN_ROWS * 32; idx += QN_COMPUTE_WARPS * 32) {
      const int r = idx >> 5, col = idx & 31;
      float u = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) u = __fadd_rn(u, red[w][r][col]);
      const int row = row_base + r;
      if (row < p.M) {
        const float uf = __fmul_rn(u, p.lora_scale);  // also undoes 2^-e
        const __nv_bfloat16 hi = __float2bfloat16_rn(uf);
        const __nv_bfloat16 lo = __float2bfloat16_rn(__fsub_rn(uf, __bfloat162float(hi)));
        uint16_t* la = p.lora_act + (size_t)row * 64;
        la[col] = __bfloat16_as_ushort(hi);
        la[32 + col] = __bfloat16_as_ushort(lo);
      }
    }
  }
}

}  // namespace

cudaError_t launch_quantize_nvfp4(const QuantActParams& p, const CUtensorMap& tm_x, const CUtensorMap& tm_l1t,
                                  int* dev_status, unsigned long long timeout_ns, cudaStream_t stream, bool pdl) {
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e =
        cudaFuncSetAttribute(quantize_nvfp4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)QN_SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.M_pad / QN_ROWS);  // covers the scale padding rows (zero scales)
  cfg.blockDim = dim3(QN_THREADS);
  cfg.dynamicSmemBytes = QN_SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  set_pdl(cfg, attr, pdl);
  return cudaLaunchKernelEx(&cfg, quantize_nvfp4_kernel, tm_x, tm_l1t, p, dev_status, timeout_ns);
}

}  // namespace svdq
