// S2 on CTA pairs: the W4A4 NVFP4 GEMM with the low-rank up-projection and
// bias in its epilogue, one M = 256 MMA per pair of SMs (tcgen05
// .cta_group::2).
//
// Page: "Hugging Face integrates Nunchaku 4-bit diffusion inference into
// Diffusers", section "SVDQuant and the Nunchaku engine": the engine fuses the
// low-rank up-projection into the 4-bit GEMM.  Same arithmetic as the
// single-CTA kernel (gemm_nvfp4.cu):
//
//   D  = sum_k E2M1(a) E4M3(sfa) * E2M1(b) E4M3(sfb)      (kind::mxf4nvf4)
//      + [hi(u/alpha) | lo(u/alpha)] . [L2^T|L2^T]        (kind::f16, same D)
//   y  = bf16(alpha * D + bias),   alpha = s_a * s_w
//
// Why pairs: the single-CTA kernel streams 54 KB of operands per K slice into
// every SM and is bound by that load ring, not by the tensor cores.  Here a
// cluster of two CTAs computes a 256 x 256 output tile: CTA r holds rows
// [128 r, 128 r + 128) of the A tile and rows [128 r, 128 r + 128) of the B
// tile (half of N), the tensor cores of the two SMs exchange the B halves,
// and each CTA accumulates its 128 rows x all 256 columns in its own tensor
// memory.  Per SM and K slice that is A 16 KB + B 16 KB + scales 6 KB = 38 KB,
// so five stages fit where four did.  Each CTA needs the scales of its own A
// rows and of all 256 B rows (the block-scale layout of the M = 128 half).
//
// Roles (9 warps per CTA; the MMA and scale-copy warps are idle in CTA 1):
//   warp 0      TMA producer, both CTAs: loads into its own shared memory,
//               completion bytes counted on CTA 0's full barrier
//   warp 1      CTA 0: MMA issuer for the pair
//   warps 2..5  epilogue, both CTAs: own accumulator rows -> bf16 -> TMA store
//   warps 6..8  CTA 0: block-scale copies smem -> TMEM for both CTAs
//               (tcgen05.cp .cta_group::2), one K slice ahead of the MMAs
// Synchronisation across the pair:
//   full[s]     CTA 0 only; CTA 0's producer arms it with both CTAs' bytes
//   empty[s]    both CTAs; the MMA warp's commit multicasts to both
//   acc_full    both CTAs; multicast commit after a tile's last MMA
//   acc_empty   CTA 0 only; the epilogue warps of both CTAs arrive on it
// Tensor memory per CTA as in the single-CTA kernel: accumulators at columns
// 0 and 160 (96 shared), two 48-column scale buffers at 416 and 464.
// Every mbarrier wait is bounded; on timeout the kernel records a status code,
// drains what it can observe, and both CTAs meet at the final cluster barrier.
#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"
#include "svdq_internal.h"

namespace svdq {
namespace {

constexpr int BM = 128;                           // rows per CTA
constexpr int BN = 256;                           // output columns per tile
constexpr int BN_HALF = BN / 2;                   // B rows per CTA
constexpr int BK_BYTES = 128;                     // 256 fp4 elements per K slice
constexpr int STAGES = 5;
constexpr int A_BYTES = BM * BK_BYTES;            // 16 KB
constexpr int B_BYTES = BN_HALF * BK_BYTES;       // 16 KB
constexpr int SFA_BYTES = 4 * 512;                // 4 K64 chunks x 128 rows
constexpr int SFB_BYTES = 2 * SFA_BYTES;          // both 128-row blocks of the tile's 256 B rows
constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;  // 38 KB
static_assert(STAGE_BYTES % 1024 == 0, "stages keep the 1024-byte alignment of SWIZZLE_128B");
constexpr int EPI_WARPS = 4;
constexpr int EPI_CHUNK = 16;                     // columns per TMA store
constexpr int EPI_BUF_BYTES = 32 * EPI_CHUNK * 2;
constexpr int EPI_BYTES = EPI_WARPS * 2 * EPI_BUF_BYTES;
constexpr int SF_WARPS = 3;
constexpr int SF_WARP0 = 2 + EPI_WARPS;
constexpr int NUM_THREADS = (2 + EPI_WARPS + SF_WARPS) * 32;
constexpr int TMEM_COLS = 512;
constexpr int ACC_STRIDE = 160;
constexpr int ACC_OVERLAP = 2 * 256 - (ACC_STRIDE + 256);
constexpr int SF_COLS = 48;
constexpr int TMEM_SF0 = ACC_STRIDE + 256;
constexpr int TMEM_SFA_OFF = 0, TMEM_SFB_OFF = 16;
static_assert(TMEM_SF0 + 2 * SF_COLS <= TMEM_COLS, "two scale buffers above the accumulators");
constexpr uint16_t PAIR_MASK = 0x3;
constexpr unsigned long long kDrainLimitNs = 2000000000ull;

struct SmemCtl {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t acc_full;
  uint64_t acc_empty;
  uint64_t sf_full[2];
  uint64_t sf_empty[2];
  uint64_t drain;
  uint64_t sf_drain;
  uint32_t tmem_base;
  int abort_flag;
};

constexpr size_t SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + EPI_BYTES + sizeof(SmemCtl);

// Instruction descriptors for M = 256 (the pair), N = 256.
constexpr uint32_t IDESC_NVFP4 = (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(256 >> 4) << 24);
constexpr uint32_t IDESC_BF16 =
    (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(256 >> 4) << 24);

SVDQ_DEV uint64_t sw128_desc(uint32_t saddr) { return smem_desc(saddr, 16, 1024, 2); }
SVDQ_DEV uint64_t sf_desc(uint32_t saddr) { return smem_desc(saddr, 0, 128, 0); }

__global__ void __launch_bounds__(NUM_THREADS, 1)
    gemm_nvfp4_pair_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                           const __grid_constant__ CUtensorMap tm_la, const __grid_constant__ CUtensorMap tm_lb,
                           const __grid_constant__ CUtensorMap tm_y, const __grid_constant__ CUtensorMap tm_sfa,
                           const __grid_constant__ CUtensorMap tm_sfb, const GemmNvfp4Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stage_base = smem;
  uint8_t* epi_base = smem + STAGES * STAGE_BYTES;
  SmemCtl* ctl = reinterpret_cast<SmemCtl*>(epi_base + EPI_BYTES);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();     // 0: leader (issues the MMAs), 1: peer
  const int pair = blockIdx.x >> 1, num_pairs = gridDim.x >> 1;
  const int tiles_m = (p.M + 2 * BM - 1) / (2 * BM);
  const int tiles_n = (p.N + BN - 1) / BN;
  const int num_tiles = tiles_m * tiles_n;
  const int k_tiles = p.K / 256;
  const int slices = k_tiles + 1;  // + the low-rank slice

  // Every CTA initialises the same barrier set; only CTA 0's full[],
  // acc_empty and scale barriers are used.
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&ctl->full[s]), 1);
      mbar_init(smem_u32(&ctl->empty[s]), 1);
    }
    mbar_init(smem_u32(&ctl->acc_full), 1);
    mbar_init(smem_u32(&ctl->acc_empty), 2 * EPI_WARPS);
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
    prefetch_tmap(&tm_sfa);
    prefetch_tmap(&tm_sfb);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(&ctl->tmem_base), TMEM_COLS);
    tmem_relinquish_pair();
  }
  // Both CTAs' barriers and tensor memory exist before either is used.
  __syncwarp();
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;

  // Inputs produced by the preceding quantize kernel become visible here.
  pdl_wait();
  // The next kernel on the stream may be scheduled from now on; it waits for
  // this grid's completion before it reads anything.
  pdl_launch_dependents();

  WaitCtx wctx{&ctl->abort_flag, p.dev_status, p.timeout_ns};

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_phase = 0;  // CTA 0: per stage, load outstanding and its parity
      bool ok = true;
      const uint64_t pol = policy_evict_last();   // every operand is re-read by other tiles
      const int kch = p.K / 64;
      for (int tile = pair; tile < num_tiles && ok; tile += num_pairs) {
        const int m0 = (tile % tiles_m) * 2 * BM + (int)rank * BM;     // this CTA's A rows
        const int n0 = (tile / tiles_m) * BN;                          // the tile's B rows
        const int nb = n0 + (int)rank * BN_HALF;                       // this CTA's half of them
        for (int kt = 0; kt < slices; ++kt) {
          if (!mbar_wait(smem_u32(&ctl->empty[stage]), phase ^ 1, wctx, kDevTimeoutProducer)) {
            ok = false;
            break;
          }
          uint8_t* sa = stage_base + stage * STAGE_BYTES;
          uint8_t* sb = sa + A_BYTES;
          uint8_t* ssfa = sb + B_BYTES;
          uint8_t* ssfb = ssfa + SFA_BYTES;
          const uint32_t full_local = smem_u32(&ctl->full[stage]);
          const uint32_t full = rank == 0 ? full_local : mapa_shared(full_local, 0);
          if (kt == 0) {
            if (rank == 0) mbar_arrive_expect_tx(full_local, 2 * (A_BYTES + B_BYTES));
            tma_load_2d_pair(smem_u32(sa), &tm_la, 0, m0, full, pol);
            tma_load_2d_pair(smem_u32(sb), &tm_lb, 0, nb, full, pol);
          } else {
            const int kb = kt - 1;
            if (rank == 0) mbar_arrive_expect_tx(full_local, 2 * STAGE_BYTES);
            tma_load_2d_pair(smem_u32(sa), &tm_a, kb * BK_BYTES, m0, full, pol);
            tma_load_2d_pair(smem_u32(sb), &tm_b, kb * BK_BYTES, nb, full, pol);
            // Scales: 256-byte rows of the tiled layout, 2 KB (8 rows) per
            // 128-row block and K slice.
            tma_load_2d_pair(smem_u32(ssfa), &tm_sfa, 0, ((m0 / 128) * kch + kb * 4) * 2, full, pol);
            tma_load_2d_pair(smem_u32(ssfb), &tm_sfb, 0, ((n0 / 128) * kch + kb * 4) * 2, full, pol);
            tma_load_2d_pair(smem_u32(ssfb + SFA_BYTES), &tm_sfb, 0, ((n0 / 128 + 1) * kch + kb * 4) * 2, full,
                             pol);
          }
          issued_mask |= 1u << stage;
          issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // CTA 0 never leaves with copies in flight into the pair's shared
      // memory: a full[] phase completes only when both CTAs' bytes landed.
      if (rank == 0) {
        volatile int never = 0;
        WaitCtx drain_ctx{&never, p.dev_status, kDrainLimitNs};
        for (int s = 0; s < STAGES; ++s)
          if (issued_mask & (1u << s))
            mbar_wait(smem_u32(&ctl->full[s]), (issued_phase >> s) & 1, drain_ctx, kDevTimeoutDrain);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ------------------------------------------------------------ MMA issuer (CTA 0)
      int stage = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      int it = 0;
      uint32_t ks = 0;  // K slices computed so far (selects the scale buffer)
      for (int tile = pair; tile < num_tiles && ok; tile += num_pairs, ++it) {
        const uint32_t d_tmem = tmem + (uint32_t)((it & 1) * ACC_STRIDE);
        // Both CTAs' epilogues have taken the shared columns of this accumulator.
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
              mma_bf16_pair(d_tmem, sw128_desc(sa + 32 * j), sw128_desc(sb + 32 * j), IDESC_BF16, j > 0 ? 1u : 0u);
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
              mma_nvfp4_pair(d_tmem, sw128_desc(sa + 32 * j), sw128_desc(sb + 32 * j), IDESC_NVFP4,
                             sf + TMEM_SFA_OFF + 4 * j, sf + TMEM_SFB_OFF + 8 * j, 1u);
            tc_commit_pair(smem_u32(&ctl->sf_empty[buf]));
            ++ks;
          }
          // Both CTAs may refill this stage once the MMAs reading it are done.
          tc_commit_pair_mc(smem_u32(&ctl->empty[stage]), PAIR_MASK);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        tc_commit_pair_mc(smem_u32(&ctl->acc_full), PAIR_MASK);
        acc_phase ^= 1;
      }
      // Wait for every MMA this thread issued before tensor memory is freed.
      tc_commit_pair(smem_u32(&ctl->drain));
      volatile int never = 0;
      WaitCtx drain_ctx{&never, p.dev_status, kDrainLimitNs};
      mbar_wait(smem_u32(&ctl->drain), 0, drain_ctx, kDevTimeoutDrain);
    }
  } else if (warp >= SF_WARP0) {
    if (lane == 0 && rank == 0) {
      // ------------------------------------------------------------ scale copies (CTA 0, for both)
      // Warp SF_WARP0 + w copies part w of every K slice's block scales in
      // both CTAs: w = 0: SFA, w = 1 / 2: SFB rows 0-127 / 128-255 of the tile.
      const int w = warp - SF_WARP0;
      int stage = 0;
      uint32_t phase = 0, ks = 0;
      bool ok = true;
      for (int tile = pair; tile < num_tiles && ok; tile += num_pairs) {
        for (int kt = 0; kt < slices; ++kt) {
          if (kt > 0) {
            const uint32_t buf = ks & 1;
            // The MMAs of the K slice two back read this buffer; wait for them.
            if (ks >= 2 && !mbar_wait(smem_u32(&ctl->sf_empty[buf]), ((ks - 2) >> 1) & 1, wctx, kDevTimeoutMma)) {
              ok = false;
              break;
            }
            // full[] completes only when both CTAs' scales have landed.
            if (!mbar_wait(smem_u32(&ctl->full[stage]), phase, wctx, kDevTimeoutMma)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t ssfa = smem_u32(stage_base + stage * STAGE_BYTES) + A_BYTES + B_BYTES;
            const uint32_t src = ssfa + SFA_BYTES * w;
            const uint32_t dst = tmem + TMEM_SF0 + buf * SF_COLS + (w == 0 ? TMEM_SFA_OFF : TMEM_SFB_OFF + 4 * (w - 1));
            const uint32_t col_step = w == 0 ? 4 : 8;
#pragma unroll
            for (int j = 0; j < 4; ++j) tmem_cp_pair_32x128_warpx4(dst + col_step * j, sf_desc(src + 512 * j));
            tc_commit_pair(smem_u32(&ctl->sf_full[buf]));
            ++ks;
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      tc_commit_pair(smem_u32(&ctl->sf_drain));
      volatile int never = 0;
      WaitCtx drain_ctx{&never, p.dev_status, kDrainLimitNs};
      mbar_wait(smem_u32(&ctl->sf_drain), 0, drain_ctx, kDevTimeoutDrain);
    }
  } else {
    // -------------------------------------------------------------- epilogue (both CTAs)
    // Each warp owns 32 rows (its TMEM lane quarter) of this CTA's 128 rows x
    // 256 columns, read from TMEM 32 columns at a time into a ring of three
    // register blocks: the chunks holding the columns shared with the other
    // accumulator first, one wait, then the release on CTA 0's acc_empty
    // (remote for CTA 1) before anything is converted.
    const int q = warp & 3;
    uint8_t* buf0 = epi_base + (warp - 2) * 2 * EPI_BUF_BYTES;
    const uint32_t acc_empty_local = smem_u32(&ctl->acc_empty);
    const uint32_t acc_empty_leader = rank == 0 ? acc_empty_local : mapa_shared(acc_empty_local, 0);
    uint32_t acc_phase = 0;
    int chunk_seq = 0, it = 0;
    constexpr int LDC = 32;
    constexpr int NCH = BN / LDC;
    constexpr int NSH = (ACC_OVERLAP + LDC - 1) / LDC;
    constexpr int NBUF = 3;
    static_assert(NSH <= NBUF, "the shared chunks fit the first ring fill");
    for (int tile = pair; tile < num_tiles; tile += num_pairs, ++it) {
      const int m0 = (tile % tiles_m) * 2 * BM + (int)rank * BM;
      const int n0 = (tile / tiles_m) * BN;
      const int b = it & 1;
      uint4 bias8 = make_uint4(0, 0, 0, 0);
      if (p.bias != nullptr && n0 + 8 * lane < p.N) bias8 = __ldg(reinterpret_cast<const uint4*>(p.bias + n0) + lane);
      const bool got = mbar_wait(smem_u32(&ctl->acc_full), acc_phase, wctx, kDevTimeoutEpilogue);
      if (!__all_sync(0xffffffffu, got)) break;  // warp-uniform decision
      tc_fence_after();
      const uint32_t acc_base = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(b * ACC_STRIDE);
      auto chunk_col = [&](int i) { return b == 0 ? (i + NCH - NSH) % NCH : i; };
      uint32_t rb[NBUF][32];
#pragma unroll
      for (int i = 0; i < NBUF; ++i) tmem_ld_32x32b_x32(acc_base + chunk_col(i) * LDC, rb[i]);
      tmem_ld_wait(rb[0]);
      reg_fence(rb[1]);
      reg_fence(rb[2]);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (rank == 0)
          mbar_arrive(acc_empty_local);
        else
          mbar_arrive_cluster(acc_empty_leader);
      }
#pragma unroll
      for (int i = 0; i < NCH; ++i) {
        uint32_t(&r)[32] = rb[i % NBUF];
        if (i >= NBUF && i % NBUF == 0) {
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
          if (lane == 0) bulk_wait_read<1>();   // the store two halves ago has read this buffer
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
        if (i + NBUF < NCH) tmem_ld_32x32b_x32(acc_base + chunk_col(i + NBUF) * LDC, r);
      }
      acc_phase ^= 1;
    }
    if (lane == 0) bulk_wait<0>();
  }

  // Both CTAs leave together: CTA 0's MMAs write CTA 1's tensor memory, and
  // CTA 1's loads count on CTA 0's barriers.
  __syncwarp();
  tc_fence_before();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, TMEM_COLS);
  }
}

}  // namespace

cudaError_t launch_gemm_nvfp4_pair(const GemmNvfp4Params& p, const GemmPairTmaps& t, cudaStream_t stream, bool pdl) {
  static int max_pairs = -1;
  if (max_pairs < 0) {
    cudaError_t e =
        cudaFuncSetAttribute(gemm_nvfp4_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t q = {};
    q.gridDim = dim3(2);
    q.blockDim = dim3(NUM_THREADS);
    q.dynamicSmemBytes = SMEM_BYTES;
    cudaLaunchAttribute ca[1];
    ca[0].id = cudaLaunchAttributeClusterDimension;
    ca[0].val.clusterDim.x = 2;
    ca[0].val.clusterDim.y = 1;
    ca[0].val.clusterDim.z = 1;
    q.attrs = ca;
    q.numAttrs = 1;
    int n = 0;
    e = cudaOccupancyMaxActiveClusters(&n, gemm_nvfp4_pair_kernel, &q);
    if (e != cudaSuccess) return e;
    if (n < 1) return cudaErrorInvalidConfiguration;
    max_pairs = n;
  }
  const int tiles = ((p.M + 255) / 256) * ((p.N + BN - 1) / BN);
  const int pairs = tiles < max_pairs ? tiles : max_pairs;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs);
  cfg.blockDim = dim3(NUM_THREADS);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, gemm_nvfp4_pair_kernel, t.a, t.b, t.la, t.lb, t.y, t.sfa, t.sfb, p);
}

}  // namespace svdq
