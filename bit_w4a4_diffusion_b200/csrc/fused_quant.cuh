// The activation side of the fused NVFP4 layer kernel: units of the
// smoothing + NVFP4 quantization + low-rank down-projection (the arithmetic
// of quantize_nvfp4.cu, bit for bit on codes and scales), run by the GEMM's
// epilogue warps while their accumulator is not ready, and the hand-off of a
// finished 128-row block to the GEMM's producer.
//
// Page: "Hugging Face integrates Nunchaku 4-bit diffusion inference into
// Diffusers", section "SVDQuant and the Nunchaku engine": the engine fuses the
// low-rank down-projection into the quantize kernel and the up-projection
// into the 4-bit GEMM; here both halves run in one kernel.
//
// Per element and unit (128 rows x K / splits columns of x):
//   x_hat = fp32(x) * inv_lambda
//   per 16 along K: a = max|x_hat|, sb = E4M3(a * fp32(1/(6 s_a))),
//     d = float(sb) * s_a, code = E2M1(x_hat * fp32(1/d))        (RNE, satfinite)
//   u_part[split] = (x_hat 2^-e in fp16) . (L1 in fp16), fp32 accumulate
// and, by the last unit of a row block:
//   lora_act = [hi | lo] of (sum over splits, in split order) * 2^e / (s_a s_w)
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "epilogue.cuh"
#include "ptx.cuh"
#include "svdq_internal.h"

namespace svdq {

// Streaming load of data read once (not kept in L1).
SVDQ_DEV uint4 ld_stream_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}
// Read-only load kept in L1 (1/lambda and L1^T, read by every unit).
SVDQ_DEV uint4 ld_ro_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}
SVDQ_DEV int ld_acquire_gpu(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
// Atomic add with acquire-release semantics at GPU scope (one round trip
// where a fence, the add and another fence would take three).
SVDQ_DEV int atomic_add_acq_rel_gpu(int* p, int v) {
  int old;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}
SVDQ_DEV void st_release_gpu(int* p, int v) {
  asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// Orders this thread's generic-proxy global accesses with later (or, on the
// writing side, other threads' later) async-proxy accesses such as TMA loads.
SVDQ_DEV void fence_proxy_async_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }
// Brings a box of a tensor into L2 (no shared memory involved, no completion).
SVDQ_DEV void prefetch_tensor_l2(const CUtensorMap* m, int x, int y) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(
                   reinterpret_cast<uint64_t>(m)),
               "r"(x), "r"(y)
               : "memory");
}

// Bounded wait until the word at `flag` is nonzero (acquire, GPU scope).
// Gives up like mbar_wait: on the CTA's abort word, or after ctx.limit_ns,
// recording `code` in the status word and raising the abort word.
SVDQ_DEV bool flag_wait(const int* flag, const WaitCtx& ctx, int code) {
  if (ld_acquire_gpu(flag) != 0) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t i = 1;; ++i) {
    if (i == 1 || (i & 15) == 0) {
      if (*ctx.abort_flag) return false;
      if (globaltimer_ns() - t0 > ctx.limit_ns) {
        *ctx.abort_flag = 1;
        if (ctx.dev_status) atomicCAS(ctx.dev_status, 0, code);
        return false;
      }
    }
    __nanosleep(100);
    if (ld_acquire_gpu(flag) != 0) return true;
  }
}

// One lane's view of a warp's 16 rows: lane (g, c) holds columns 8c..8c+7
// of every 32-column block for rows g and g + 8; those 16 values are also its
// mma.m16n8k16 A fragments under a permutation of k that the L1^T fragments
// (rank 8 j + g, the same 8 columns) follow.
struct QuantLane {
  const uint16_t* xr0;   // row g's x at column 8c (row g + 8's is 8 K further)
  const float* inv;      // 1/lambda at column 8c
  const uint16_t* l1t;   // L1^T row (rank) g at column 8c
  uint8_t* code0;        // row g's code bytes at column 8c (row g + 8's is 4 K further)
  int row0, K, c;
  bool ok0, ok1;         // rows g, g + 8 lie below M
};

struct QuantBlock {
  uint4 xa, xb, i0, i1;
};

// x of a block (from L2 or HBM: loaded two blocks ahead).
SVDQ_DEV void quant_load_x(QuantBlock& b, const QuantLane& L, int k) {
  const uint4 z = make_uint4(0u, 0u, 0u, 0u);
  b.xa = L.ok0 ? ld_stream_v4(L.xr0 + k) : z;
  b.xb = L.ok1 ? ld_stream_v4(L.xr0 + (size_t)8 * L.K + k) : z;
}
// 1/lambda of a block (the same columns for all eight warps of the unit,
// mostly L1 hits: loaded one block ahead).
SVDQ_DEV void quant_load_w(QuantBlock& b, const QuantLane& L, int k) {
  b.i0 = ld_ro_v4(L.inv + k);
  b.i1 = ld_ro_v4(L.inv + k + 4);
}

// Quantizes the 32-column block at column k of the lane's two rows (codes and
// scale bytes stored), and adds its low-rank products into acc (n-tile j:
// ranks 8 j + 2c, 8 j + 2c + 1 of rows g and g + 8).
SVDQ_DEV void quant_arith(const QuantBlock& b, const uint4 (&lf)[4], const QuantLane& L, int k, const float* rcp_tab,
                          float inv_six_s, float2 xs2, uint8_t* scales, float (&acc)[4][4]) {
  const bool odd = (L.c & 1) != 0;
  const uint32_t wa[4] = {b.xa.x, b.xa.y, b.xa.z, b.xa.w}, wb[4] = {b.xb.x, b.xb.y, b.xb.z, b.xb.w};
  const float il[8] = {__uint_as_float(b.i0.x), __uint_as_float(b.i0.y), __uint_as_float(b.i0.z),
                       __uint_as_float(b.i0.w), __uint_as_float(b.i1.x), __uint_as_float(b.i1.y),
                       __uint_as_float(b.i1.z), __uint_as_float(b.i1.w)};
  float2 v0[4], v1[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 ilp = make_float2(il[2 * i], il[2 * i + 1]);
    v0[i] = __fmul2_rn(bf16x2_to_float2(wa[i]), ilp);
    v1[i] = __fmul2_rn(bf16x2_to_float2(wb[i]), ilp);
  }
  // The group of 16 is the lane pair (c, c ^ 1).
  float a0 = 0.f, a1 = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    a0 = fmaxf(a0, fmaxf(fabsf(v0[i].x), fabsf(v0[i].y)));
    a1 = fmaxf(a1, fmaxf(fabsf(v1[i].x), fabsf(v1[i].y)));
  }
  a0 = fmaxf(a0, __shfl_xor_sync(0xffffffffu, a0, 1));
  a1 = fmaxf(a1, __shfl_xor_sync(0xffffffffu, a1, 1));
  // The even lane derives row g's scale, the odd lane row g + 8's; they swap.
  const uint32_t sb_m = cvt_e4m3(__fmul_rn(odd ? a1 : a0, inv_six_s));
  const float r_m = rcp_tab[sb_m & 0xFF];        // 0 marks an all-zero group
  const float r_o = __shfl_xor_sync(0xffffffffu, r_m, 1);
  const uint32_t sb_o = __shfl_xor_sync(0xffffffffu, sb_m, 1);
  const float q0 = odd ? r_o : r_m, q1 = odd ? r_m : r_o;
  const float2 qq0 = make_float2(q0, q0), qq1 = make_float2(q1, q1);
  const uint32_t w0 = q0 != 0.f ? cvt_e2m1x8(__fmul2_rn(v0[0], qq0), __fmul2_rn(v0[1], qq0), __fmul2_rn(v0[2], qq0),
                                             __fmul2_rn(v0[3], qq0))
                                : 0u;
  const uint32_t w1 = q1 != 0.f ? cvt_e2m1x8(__fmul2_rn(v1[0], qq1), __fmul2_rn(v1[1], qq1), __fmul2_rn(v1[2], qq1),
                                             __fmul2_rn(v1[3], qq1))
                                : 0u;
  if (L.ok0) __stcg(reinterpret_cast<unsigned int*>(L.code0 + k / 2), w0);
  if (L.ok1) __stcg(reinterpret_cast<unsigned int*>(L.code0 + (size_t)4 * L.K + k / 2), w1);
  if (!odd) {
    // Rows past M (up to the 256-row padding) get scale 0: their x is 0.
    const int grp = (k >> 4) + (L.c >> 1);
    scales[tiled_scale_offset(L.row0, grp, L.K)] = (uint8_t)sb_m;
    scales[tiled_scale_offset(L.row0 + 8, grp, L.K)] = (uint8_t)sb_o;
  }
  // Low-rank down-projection: A = x_hat * 2^-e in fp16.
  uint32_t a[2][4];
#pragma unroll
  for (int st = 0; st < 2; ++st) {
    const float2 p00 = __fmul2_rn(v0[2 * st], xs2), p01 = __fmul2_rn(v0[2 * st + 1], xs2);
    const float2 p10 = __fmul2_rn(v1[2 * st], xs2), p11 = __fmul2_rn(v1[2 * st + 1], xs2);
    a[st][0] = half2_bits(p00.x, p00.y);
    a[st][1] = half2_bits(p10.x, p10.y);
    a[st][2] = half2_bits(p01.x, p01.y);
    a[st][3] = half2_bits(p11.x, p11.y);
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    mma_16816(acc[j], a[0][0], a[0][1], a[0][2], a[0][3], lf[j].x, lf[j].y);
    mma_16816(acc[j], a[1][0], a[1][1], a[1][2], a[1][3], lf[j].z, lf[j].w);
  }
}

SVDQ_DEV void quant_block(const QuantBlock& b, const QuantLane& L, int k, const float* rcp_tab, float inv_six_s,
                          float2 xs2, uint8_t* scales, float (&acc)[4][4]) {
  // The L1^T fragments are used last (by the MMAs): loaded here, their
  // latency (L1 hits, mostly) hides behind the quantizer's arithmetic.
  uint4 lf[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) lf[j] = ld_ro_v4(L.l1t + (size_t)8 * j * L.K + k);
  quant_arith(b, lf, L, k, rcp_tab, inv_six_s, xs2, scales, acc);
}

// One warp's share of unit (rb, sp): rows 128 rb + 16 w .. + 15, columns
// [sp K / splits, (sp + 1) K / splits).  Codes and scales go to their buffers,
// the low-rank partial of the 16 rows to slot sp of u_part.  Loads run two
// 32-column blocks ahead of the arithmetic.
SVDQ_DEV void quant_unit(const FusedQuantParams& q, int M, int K, int rb, int sp, int w, int lane,
                         const float* rcp_tab) {
  const int g = lane >> 2, c = lane & 3;
  QuantLane L;
  L.row0 = rb * 128 + 16 * w + g;
  L.K = K;
  L.c = c;
  L.ok0 = L.row0 < M;
  L.ok1 = L.row0 + 8 < M;
  L.xr0 = q.x + (size_t)L.row0 * K + 8 * c;          // dereferenced only below M
  L.code0 = q.codes + (size_t)L.row0 * (K / 2) + 4 * c;
  L.inv = q.inv_smooth + 8 * c;
  L.l1t = q.l1t + (size_t)g * K + 8 * c;
  const float inv_six_s = __frcp_rn(__fmul_rn(6.0f, q.act_scale));
  const float2 xs2 = make_float2(q.lr_in_scale, q.lr_in_scale);
  float acc[4][4];
#pragma unroll
  for (int j = 0; j < 4; ++j)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[j][e] = 0.f;
  const int span = K / q.splits, k0 = sp * span, nb = span / 32;
  // Two rotating buffers, unrolled by two so that none is copied: x and
  // 1/lambda one block ahead.
  QuantBlock b0, b1;
  auto kb = [&](int i) { return k0 + 32 * i; };
  quant_load_x(b0, L, kb(0));
  quant_load_w(b0, L, kb(0));
  for (int i = 0; i < nb; i += 2) {
    if (i + 1 < nb) {
      quant_load_x(b1, L, kb(i + 1));
      quant_load_w(b1, L, kb(i + 1));
    }
    quant_block(b0, L, kb(i), rcp_tab, inv_six_s, xs2, q.scales, acc);
    if (i + 1 >= nb) break;
    if (i + 2 < nb) {
      quant_load_x(b0, L, kb(i + 2));
      quant_load_w(b0, L, kb(i + 2));
    }
    quant_block(b1, L, kb(i + 1), rcp_tab, inv_six_s, xs2, q.scales, acc);
  }
  const size_t mp = (size_t)q.row_blocks * 128;
  float* u0 = q.u_part + ((size_t)sp * mp + L.row0) * 32 + 2 * c;
  float* u1 = u0 + 8 * 32;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    __stcg(reinterpret_cast<float2*>(u0 + 8 * j), make_float2(acc[j][0], acc[j][1]));
    __stcg(reinterpret_cast<float2*>(u1 + 8 * j), make_float2(acc[j][2], acc[j][3]));
  }
}

// ---------------------------------------------------------------- TMA-fed units
// A unit's columns arrive in chunks of 64 through a two-buffer ring in shared
// memory, each buffer holding x [128 rows x 64] and L1^T [32 ranks x 64] as
// 64-wide SWIZZLE_128B boxes and 1/lambda [64] (fp32).  Warp w takes rows
// 16 w + perm(g), + 8 (perm = 0 4 1 5 2 6 3 7: the 128-byte swizzle puts rows
// r and r + 1 in the same bank groups, so the two rows of a quarter-warp
// load differ in bit 2), and L1^T ranks 8 j + perm(g) for its B fragments:
// accumulator columns 2c, 2c + 1 of n-tile j are then ranks 8 j + c and
// 8 j + 4 + c.
constexpr int QC_COLS = 64;                          // columns per chunk
constexpr int QC_X_BYTES = 128 * 128;                // x box: 128 rows of 128 bytes
constexpr int QC_L_BYTES = 32 * 128;                 // L1^T box: 32 ranks of 128 bytes
constexpr int QC_I_BYTES = QC_COLS * 4;              // 1/lambda
constexpr int QC_BUF_BYTES = QC_X_BYTES + QC_L_BYTES + 1024;   // 1/lambda padded to 1 KB
constexpr int QC_TX_BYTES = QC_X_BYTES + QC_L_BYTES + QC_I_BYTES;

SVDQ_DEV int quant_perm(int g) { return ((g & 1) << 2) | (g >> 1); }

// Shared-memory address of the 16-byte chunk j (elements 8j..8j+7) of row r
// in a 64-wide SWIZZLE_128B box.
SVDQ_DEV uint32_t sw128_chunk_addr(uint32_t box, int r, int j) {
  return box + (uint32_t)r * 128u + (uint32_t)((j ^ (r & 7)) << 4);
}

SVDQ_DEV uint4 lds_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

// One chunk (columns k .. k + 63) for the warp's two rows per lane, from the
// buffer at `buf`.  r0 is the lane's first row within the unit's 128.
SVDQ_DEV void quant_chunk(uint32_t buf, int k, const QuantLane& L, int r0, const float* rcp_tab, float inv_six_s,
                          float2 xs2, uint8_t* scales, float (&acc)[4][4]) {
  const int g = (threadIdx.x & 31) >> 2;
  const int pg = quant_perm(g);
#pragma unroll
  for (int blk = 0; blk < 2; ++blk) {
    const int chunk = blk * 4 + L.c;                     // 16-byte chunk of the lane in the 128-byte row
    QuantBlock b;
    b.xa = lds_v4(sw128_chunk_addr(buf, r0, chunk));
    b.xb = lds_v4(sw128_chunk_addr(buf, r0 + 8, chunk));
    const uint32_t ia = buf + QC_X_BYTES + QC_L_BYTES + (uint32_t)(blk * 32 + 8 * L.c) * 4;
    b.i0 = lds_v4(ia);
    b.i1 = lds_v4(ia + 16);
    uint4 lf[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) lf[j] = lds_v4(sw128_chunk_addr(buf + QC_X_BYTES, 8 * j + pg, chunk));
    quant_arith(b, lf, L, k + 32 * blk, rcp_tab, inv_six_s, xs2, scales, acc);
  }
}

// The last unit of row block rb: thread t (0..255) adds the splits' partials
// of row 128 rb + t / 2, ranks 16 (t % 2) .. + 15, in split order, and writes
// that row's [hi | lo] low-rank activation.
SVDQ_DEV void reduce_row_block(const FusedQuantParams& q, int M, int rb, int t) {
  const int row = rb * 128 + (t >> 1), h = t & 1;
  const size_t mp = (size_t)q.row_blocks * 128;
  float s[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) s[i] = 0.f;
  for (int sp = 0; sp < q.splits; ++sp) {
    const float4* src = reinterpret_cast<const float4*>(q.u_part + ((size_t)sp * mp + row) * 32 + 16 * h);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 v = __ldcg(src + i);
      s[4 * i] = __fadd_rn(s[4 * i], v.x);
      s[4 * i + 1] = __fadd_rn(s[4 * i + 1], v.y);
      s[4 * i + 2] = __fadd_rn(s[4 * i + 2], v.z);
      s[4 * i + 3] = __fadd_rn(s[4 * i + 3], v.w);
    }
  }
  if (row >= M) return;
  uint32_t hi[8], lo[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float u0 = __fmul_rn(s[2 * i], q.lora_scale), u1 = __fmul_rn(s[2 * i + 1], q.lora_scale);
    const __nv_bfloat16 h0 = __float2bfloat16_rn(u0), h1 = __float2bfloat16_rn(u1);
    const __nv_bfloat16 l0 = __float2bfloat16_rn(__fsub_rn(u0, __bfloat162float(h0)));
    const __nv_bfloat16 l1 = __float2bfloat16_rn(__fsub_rn(u1, __bfloat162float(h1)));
    hi[i] = (uint32_t)__bfloat16_as_ushort(h0) | ((uint32_t)__bfloat16_as_ushort(h1) << 16);
    lo[i] = (uint32_t)__bfloat16_as_ushort(l0) | ((uint32_t)__bfloat16_as_ushort(l1) << 16);
  }
  uint4* dst = reinterpret_cast<uint4*>(q.lora_act + (size_t)row * 64 + 16 * h);
  __stcg(dst, make_uint4(hi[0], hi[1], hi[2], hi[3]));
  __stcg(dst + 1, make_uint4(hi[4], hi[5], hi[6], hi[7]));
  __stcg(dst + 4, make_uint4(lo[0], lo[1], lo[2], lo[3]));      // column 32 + 16 h
  __stcg(dst + 5, make_uint4(lo[4], lo[5], lo[6], lo[7]));
}

}  // namespace svdq
