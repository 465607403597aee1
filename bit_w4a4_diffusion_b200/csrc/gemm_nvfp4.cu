// S2: the W4A4 NVFP4 GEMM with the low-rank up-projection and bias in its
// epilogue, on 5th-generation tensor cores.
//
// Page: "Hugging Face integrates Nunchaku 4-bit diffusion inference into
// Diffusers", section "SVDQuant and the Nunchaku engine": the engine fuses the
// low-rank up-projection into the 4-bit GEMM.  Here the fusion is exact
// accumulator sharing:
//
//   D  = sum_k E2M1(a) E4M3(sfa) * E2M1(b) E4M3(sfb)      (kind::mxf4nvf4)
//      + [hi(u/alpha) | lo(u/alpha)] . [L2^T | L2^T]        (kind::f16, same D)
//   y  = bf16(alpha * D + bias),   alpha = s_a * s_w
//
// so the rank-r branch is four extra bf16 MMAs into the same TMEM accumulator
// and the epilogue is a single fused multiply-add per element.
//
// Structure: persistent CTAs, one 128x256 output tile at a time, 9 warps:
//   warp 0      TMA producer (A/B codes by tensor TMA, scales by bulk copy)
//   warp 1      MMA issuer (MMAs and commits only)
//   warps 2..5  epilogue (TMEM -> registers -> bf16 -> swizzled smem -> TMA store)
//   warps 6..8  block-scale copies smem -> TMEM (SFA, SFB rows 0-127, SFB rows
//               128-255), running ahead of the MMA warp into a second buffer.
//               Copies issued by the MMA thread itself would be ordered with
//               its MMAs for free, but each one takes tens of cycles of the
//               tensor pipe (about 40 on sm_100a, only about three per four
//               MMAs hide); issued from other threads they overlap the MMAs.
// Pipeline: STAGES-deep smem ring of K=256 slices; slot 0 of every tile is the
// low-rank slice (u' in the A slot, [L2^T|L2^T] in the B slot).
// Tensor memory (512 columns): two 256-column fp32 accumulators at columns 0
// and 160, overlapping in [160, 256), and two 48-column block-scale buffers
// in [416, 512) (K slices alternate buffers).  Consecutive tiles alternate
// accumulators; the epilogue loads the 96 shared columns into registers first
// and releases the accumulator at once, so the next tile's MMAs run while the
// epilogue converts and stores.
// Every mbarrier wait is bounded; on timeout the kernel records a status code,
// drains its in-flight copies and MMAs, frees TMEM and returns.
#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"
#include "svdq_internal.h"

namespace svdq {
namespace {

constexpr int BM = 128, BN = 256;
constexpr int BK_BYTES = 128;  // 256 fp4 elements
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK_BYTES;            // 16 KB
constexpr int B_BYTES = BN * BK_BYTES;            // 32 KB
constexpr int SFA_BYTES = 4 * 512;                // 4 K64 chunks x 128 rows
constexpr int SFB_BYTES = 2 * 4 * 512;            // 2 row blocks
constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;  // 54 KB
constexpr int EPI_WARPS = 4;
constexpr int EPI_CHUNK = 16;                          // columns per TMEM load / store
constexpr int EPI_BUF_BYTES = 32 * EPI_CHUNK * 2;      // 32 rows x 32 B
constexpr int EPI_BYTES = EPI_WARPS * 2 * EPI_BUF_BYTES;
constexpr int SF_WARPS = 3;
constexpr int SF_WARP0 = 2 + EPI_WARPS;                 // first scale-copy warp
constexpr int NUM_THREADS = (2 + EPI_WARPS + SF_WARPS) * 32;
constexpr int TMEM_COLS = 512;
constexpr int ACC_STRIDE = 160;                        // accumulator b starts at column b * 160
constexpr int ACC_OVERLAP = 2 * 256 - (ACC_STRIDE + 256); // 96 shared columns
// Block scales of one K slice: SFA 4 MMAs x 4 columns, SFB 4 MMAs x 8 columns.
constexpr int SF_COLS = 48;
constexpr int TMEM_SF0 = ACC_STRIDE + 256;             // buffers at 416 and 464
constexpr int TMEM_SFA_OFF = 0, TMEM_SFB_OFF = 16;
// Limit for the exit-path waits on this CTA's own in-flight copies and MMAs,
// which always complete; independent of the caller's timeout.
constexpr unsigned long long kDrainLimitNs = 2000000000ull;

struct SmemCtl {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t acc_full;
  uint64_t acc_empty;
  uint64_t sf_full[2];   // scale-copy warps -> MMA (copies of one K slice landed)
  uint64_t sf_empty[2];  // MMA -> scale-copy warps (MMAs reading the buffer done)
  uint64_t drain;
  uint64_t sf_drain;
  uint32_t tmem_base;
  int abort_flag;
};

constexpr size_t SMEM_BYTES = 1024 /*align slack*/ + STAGES * STAGE_BYTES + EPI_BYTES + sizeof(SmemCtl);

// Instruction descriptors (tcgen05 "instruction descriptor" bit fields).
//   block-scaled: a/b format E2M1 (=1) at bits 7/10, N>>3 at 17, UE4M3 scales
//   (bit 23 = 0), M>>4 at 24.  f16 kind: f32 accumulate (bit 4), bf16 a/b (=1).
constexpr uint32_t IDESC_NVFP4 = (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
constexpr uint32_t IDESC_BF16 =
    (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);

SVDQ_DEV uint64_t sw128_desc(uint32_t saddr) { return smem_desc(saddr, 16, 1024, 2); }
SVDQ_DEV uint64_t sf_desc(uint32_t saddr) { return smem_desc(saddr, 0, 128, 0); }

__global__ void __launch_bounds__(NUM_THREADS, 1)
    gemm_nvfp4_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                      const __grid_constant__ CUtensorMap tm_la, const __grid_constant__ CUtensorMap tm_lb,
                      const __grid_constant__ CUtensorMap tm_y, const GemmNvfp4Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stage_base = smem;
  uint8_t* epi_base = smem + STAGES * STAGE_BYTES;
  SmemCtl* ctl = reinterpret_cast<SmemCtl*>(epi_base + EPI_BYTES);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles_m = (p.M + BM - 1) / BM;
  const int tiles_n = (p.N + BN - 1) / BN;
  const int num_tiles = tiles_m * tiles_n;
  const int k_tiles = p.K / 256;
  const int slices = k_tiles + 1;  // + the low-rank slice

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&ctl->full[s]), 1);
      mbar_init(smem_u32(&ctl->empty[s]), 1);
    }
    mbar_init(smem_u32(&ctl->acc_full), 1);
    mbar_init(smem_u32(&ctl->acc_empty), EPI_WARPS);
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&ctl->sf_full[b]), SF_WARPS);
      mbar_init(smem_u32(&ctl->sf_empty[b]), 1);
    }
    mbar_init(smem_u32(&ctl->drain), 1);
    mbar_init(smem_u32(&ctl->sf_drain), SF_WARPS);
    ctl->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_a);
    prefetch_tmap(&tm_b);
    prefetch_tmap(&tm_la);
    prefetch_tmap(&tm_lb);
    prefetch_tmap(&tm_y);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&ctl->tmem_base), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;

  // Inputs produced by the preceding quantize kernel become visible here.
  pdl_wait();

  WaitCtx wctx{&ctl->abort_flag, p.dev_status, p.timeout_ns};

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_phase = 0;  // per stage: load outstanding, its parity
      bool ok = true;
      const uint64_t pol_w = policy_evict_last();
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const int m0 = (tile % tiles_m) * BM;
        const int n0 = (tile / tiles_m) * BN;
        for (int kt = 0; kt < slices; ++kt) {
          if (!mbar_wait(smem_u32(&ctl->empty[stage]), phase ^ 1, wctx, kDevTimeoutProducer)) {
            ok = false;
            break;
          }
          uint8_t* sa = stage_base + stage * STAGE_BYTES;
          uint8_t* sb = sa + A_BYTES;
          uint8_t* ssfa = sb + B_BYTES;
          uint8_t* ssfb = ssfa + SFA_BYTES;
          const uint32_t full = smem_u32(&ctl->full[stage]);
          if (kt == 0) {
            mbar_arrive_expect_tx(full, A_BYTES + B_BYTES);
            tma_load_2d(smem_u32(sa), &tm_la, 0, m0, full);
            tma_load_2d_hint(smem_u32(sb), &tm_lb, 0, n0, full, pol_w);
          } else {
            const int kb = kt - 1;
            mbar_arrive_expect_tx(full, STAGE_BYTES);
            tma_load_2d(smem_u32(sa), &tm_a, kb * BK_BYTES, m0, full);
            tma_load_2d_hint(smem_u32(sb), &tm_b, kb * BK_BYTES, n0, full, pol_w);
            const size_t kch = (size_t)(p.K / 64);
            bulk_load(smem_u32(ssfa), p.act_scales + ((size_t)(m0 / 128) * kch + kb * 4) * 512, SFA_BYTES, full);
            bulk_load(smem_u32(ssfb), p.w_scales + ((size_t)(n0 / 128) * kch + kb * 4) * 512, SFA_BYTES, full);
            bulk_load(smem_u32(ssfb + SFA_BYTES), p.w_scales + ((size_t)(n0 / 128 + 1) * kch + kb * 4) * 512,
                      SFA_BYTES, full);
          }
          issued_mask |= 1u << stage;
          issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // Never leave with copies in flight into this CTA's shared memory.
      volatile int never = 0;
      WaitCtx drain_ctx{&never, p.dev_status, kDrainLimitNs};
      for (int s = 0; s < STAGES; ++s)
        if (issued_mask & (1u << s))
          mbar_wait(smem_u32(&ctl->full[s]), (issued_phase >> s) & 1, drain_ctx, kDevTimeoutDrain);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      int stage = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      int it = 0;
      uint32_t ks = 0;  // K slices computed so far (selects the scale buffer)
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++it) {
        const uint32_t d_tmem = tmem + (uint32_t)((it & 1) * ACC_STRIDE);
        if (!mbar_wait(smem_u32(&ctl->acc_empty), acc_phase ^ 1, wctx, kDevTimeoutMma)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int kt = 0; kt < slices; ++kt) {
          if (!mbar_wait(smem_u32(&ctl->full[stage]), phase, wctx, kDevTimeoutMma)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(stage_base + stage * STAGE_BYTES);
          const uint32_t sb = sa + A_BYTES;
          if (kt == 0) {
#pragma unroll
            for (int j = 0; j < 4; ++j)
              mma_bf16(d_tmem, sw128_desc(sa + 32 * j), sw128_desc(sb + 32 * j), IDESC_BF16, j > 0 ? 1u : 0u);
          } else {
            const uint32_t buf = ks & 1;
            if (!mbar_wait(smem_u32(&ctl->sf_full[buf]), (ks >> 1) & 1, wctx, kDevTimeoutMma)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t sf = tmem + TMEM_SF0 + buf * SF_COLS;
#pragma unroll
            for (int j = 0; j < 4; ++j)
              mma_nvfp4(d_tmem, sw128_desc(sa + 32 * j), sw128_desc(sb + 32 * j), IDESC_NVFP4,
                        sf + TMEM_SFA_OFF + 4 * j, sf + TMEM_SFB_OFF + 8 * j, 1u);
            tc_commit(smem_u32(&ctl->sf_empty[buf]));
            ++ks;
          }
          tc_commit(smem_u32(&ctl->empty[stage]));
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        tc_commit(smem_u32(&ctl->acc_full));
        acc_phase ^= 1;
      }
      // Wait for every MMA / copy this thread issued before TMEM is freed.
      tc_commit(smem_u32(&ctl->drain));
      volatile int never = 0;
      WaitCtx drain_ctx{&never, p.dev_status, kDrainLimitNs};
      mbar_wait(smem_u32(&ctl->drain), 0, drain_ctx, kDevTimeoutDrain);
    }
  } else if (warp >= SF_WARP0) {
    if (lane == 0) {
      // ------------------------------------------------------------ scale copies
      // Warp SF_WARP0 + w copies part w of every K slice's block scales:
      // w = 0: SFA (4 copies), w = 1 / 2: SFB rows 0-127 / 128-255 (4 each).
      const int w = warp - SF_WARP0;
      int stage = 0;
      uint32_t phase = 0, ks = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        for (int kt = 0; kt < slices; ++kt) {
          if (kt > 0) {
            const uint32_t buf = ks & 1;
            // The MMAs of the K slice two back read this buffer; wait for them.
            if (ks >= 2 && !mbar_wait(smem_u32(&ctl->sf_empty[buf]), ((ks - 2) >> 1) & 1, wctx, kDevTimeoutMma)) {
              ok = false;
              break;
            }
            if (!mbar_wait(smem_u32(&ctl->full[stage]), phase, wctx, kDevTimeoutMma)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t ssfa = smem_u32(stage_base + stage * STAGE_BYTES) + A_BYTES + B_BYTES;
            const uint32_t src = w == 0 ? ssfa : ssfa + SFA_BYTES * w;
            const uint32_t dst = tmem + TMEM_SF0 + buf * SF_COLS + (w == 0 ? TMEM_SFA_OFF : TMEM_SFB_OFF + 4 * (w - 1));
            const uint32_t col_step = w == 0 ? 4 : 8;
#pragma unroll
            for (int j = 0; j < 4; ++j) tmem_cp_32x128_warpx4(dst + col_step * j, sf_desc(src + 512 * j));
            tc_commit(smem_u32(&ctl->sf_full[buf]));
            ++ks;
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      tc_commit(smem_u32(&ctl->sf_drain));
      volatile int never = 0;
      WaitCtx drain_ctx{&never, p.dev_status, kDrainLimitNs};
      mbar_wait(smem_u32(&ctl->sf_drain), 0, drain_ctx, kDevTimeoutDrain);
    }
  } else {
    // -------------------------------------------------------------- epilogue
    // Each warp owns 32 rows (its TMEM lane quarter) x 256 columns of a tile,
    // read from TMEM 32 columns at a time into a ring of three register
    // blocks.  The three chunks holding the columns shared with the other
    // accumulator are loaded first, with one wait, and the accumulator is
    // released before any of them is converted; later chunks are loaded into
    // the block just converted, three chunks ahead.  The tile's bias is loaded
    // once (lane l holds columns 8l..8l+7) and broadcast by shuffles.
    const int q = warp & 3;
    uint8_t* buf0 = epi_base + (warp - 2) * 2 * EPI_BUF_BYTES;
    uint32_t acc_phase = 0;
    int chunk_seq = 0, it = 0;
    constexpr int LDC = 32;                    // columns per TMEM load
    constexpr int NCH = BN / LDC;
    constexpr int NSH = (ACC_OVERLAP + LDC - 1) / LDC;  // chunks holding shared columns
    constexpr int NBUF = 3;
    static_assert(NSH <= NBUF, "the shared chunks fit the first ring fill");
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++it) {
      const int m0 = (tile % tiles_m) * BM;
      const int n0 = (tile / tiles_m) * BN;
      const int b = it & 1;
      uint4 bias8 = make_uint4(0, 0, 0, 0);
      if (p.bias != nullptr && n0 + 8 * lane < p.N) bias8 = __ldg(reinterpret_cast<const uint4*>(p.bias + n0) + lane);
      const bool got = mbar_wait(smem_u32(&ctl->acc_full), acc_phase, wctx, kDevTimeoutEpilogue);
      if (!__all_sync(0xffffffffu, got)) break;  // warp-uniform decision
      tc_fence_after();
      const uint32_t acc_base = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(b * ACC_STRIDE);
      // The columns shared with the other accumulator go first: the last
      // ACC_OVERLAP of accumulator 0, the first ACC_OVERLAP of accumulator 1.
      auto chunk_col = [&](int i) { return b == 0 ? (i + NCH - NSH) % NCH : i; };
      uint32_t rb[NBUF][32];
#pragma unroll
      for (int i = 0; i < NBUF; ++i) tmem_ld_32x32b_x32(acc_base + chunk_col(i) * LDC, rb[i]);
      tmem_ld_wait(rb[0]);
      reg_fence(rb[1]);
      reg_fence(rb[2]);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&ctl->acc_empty));
#pragma unroll
      for (int i = 0; i < NCH; ++i) {
        uint32_t(&r)[32] = rb[i % NBUF];
        if (i >= NBUF && i % NBUF == 0) {
          // Chunks loaded since the last wait (i .. i+2 at most) land here.
          tmem_ld_wait(rb[0]);
          reg_fence(rb[1]);
          reg_fence(rb[2]);
        }
        const int cc = chunk_col(i);
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {      // two 16-column halves per TMEM load
          const int ncol = n0 + cc * LDC + hh * EPI_CHUNK;
          const int src_lane = (cc * LDC + hh * EPI_CHUNK) / 8;  // lanes src_lane, src_lane + 1
          uint32_t bw[8];
          bw[0] = __shfl_sync(0xffffffffu, bias8.x, src_lane);
          bw[1] = __shfl_sync(0xffffffffu, bias8.y, src_lane);
          bw[2] = __shfl_sync(0xffffffffu, bias8.z, src_lane);
          bw[3] = __shfl_sync(0xffffffffu, bias8.w, src_lane);
          bw[4] = __shfl_sync(0xffffffffu, bias8.x, src_lane + 1);
          bw[5] = __shfl_sync(0xffffffffu, bias8.y, src_lane + 1);
          bw[6] = __shfl_sync(0xffffffffu, bias8.z, src_lane + 1);
          bw[7] = __shfl_sync(0xffffffffu, bias8.w, src_lane + 1);
          uint32_t packed[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const float b0 = __uint_as_float(bw[k] << 16), b1 = __uint_as_float(bw[k] & 0xFFFF0000u);
            const float y0 = __fmaf_rn(p.alpha, __uint_as_float(r[hh * 16 + 2 * k]), b0);
            const float y1 = __fmaf_rn(p.alpha, __uint_as_float(r[hh * 16 + 2 * k + 1]), b1);
            __nv_bfloat162 h2 = __floats2bfloat162_rn(y0, y1);
            packed[k] = *reinterpret_cast<uint32_t*>(&h2);
          }
          uint8_t* buf = buf0 + (chunk_seq & 1) * EPI_BUF_BYTES;
          // The TMA store issued two halves ago read this buffer; wait for it.
          if (lane == 0) bulk_wait_read<1>();
          __syncwarp();
          uint8_t* row = buf + lane * 32;
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const int pj = j ^ ((lane >> 2) & 1);  // 32-byte swizzle
            *reinterpret_cast<uint4*>(row + pj * 16) =
                make_uint4(packed[4 * j], packed[4 * j + 1], packed[4 * j + 2], packed[4 * j + 3]);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0 && ncol < p.N && m0 + 32 * q < p.M) tma_store_2d(&tm_y, ncol, m0 + 32 * q, smem_u32(buf));
          if (lane == 0) bulk_commit();
          ++chunk_seq;
        }
        // Refill the block just converted with the chunk three ahead; the
        // accumulator is still this tile's until the MMA warp reuses it, and
        // the non-shared chunks are not written by the next tile.
        if (i + NBUF < NCH) tmem_ld_32x32b_x32(acc_base + chunk_col(i + NBUF) * LDC, r);
      }
      acc_phase ^= 1;
    }
    if (lane == 0) bulk_wait<0>();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace

cudaError_t launch_gemm_nvfp4(const GemmNvfp4Params& p, const GemmTmaps& t, int num_sms, cudaStream_t stream,
                              bool pdl) {
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e =
        cudaFuncSetAttribute(gemm_nvfp4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const int tiles = ((p.M + BM - 1) / BM) * ((p.N + BN - 1) / BN);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(tiles < num_sms ? tiles : num_sms);
  cfg.blockDim = dim3(NUM_THREADS);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, gemm_nvfp4_kernel, t.a, t.b, t.la, t.lb, t.y, p);
}

}  // namespace svdq
