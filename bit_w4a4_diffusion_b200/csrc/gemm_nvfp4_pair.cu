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
// A cluster of two CTAs computes a 256 x 256 output tile: CTA r holds rows
// [128 r, 128 r + 128) of the A tile and rows [128 r, 128 r + 128) of the B
// tile (half of N), the tensor cores of the two SMs exchange the B halves,
// and each CTA accumulates its 128 rows x all 256 columns in its own tensor
// memory.  Per SM and K slice that is A 16 KB + B 16 KB + scales 6 KB = 38 KB
// of operands, against 54 KB for a 128 x 256 tile on one SM.
//
// Tensor memory (512 columns per CTA) holds ONE accumulator (columns 0-255)
// and one 48-column block-scale buffer per shared-memory stage (columns 256 +
// 48 s).  The MMA warp copies a stage's scales into its buffer itself, right
// before the MMAs that read them (tcgen05.cp then tcgen05.mma from the same
// thread are executed in order; no barrier between them).  Tying the buffer
// to the stage makes the copy safe without any wait either: a stage is
// refilled only after the MMAs that read it, and its scale buffer, have
// completed.  The price is the single accumulator: the MMAs of the next tile
// start once the eight epilogue warps of both CTAs have pulled all 256
// columns into registers, which they do with four loads each, one wait, and
// an immediate release (about 0.3 us after the tile's last MMA completes).
//
// Every role loop runs on a whole warp and issues from one elected lane: the
// tcgen05 and TMA instructions take uniform-register operands, and a loop
// run by lane 0 alone keeps its addresses in per-thread registers, which
// made each issue several times slower and the MMA warp, not the tensor
// pipe, the bottleneck.
//
// Roles (10 warps per CTA; the MMA warp is idle in CTA 1):
//   warps 0..7  epilogue, both CTAs: warp w reads TMEM lane quarter w % 4,
//               columns [128 (w / 4), + 128) -> bf16 -> TMA store
//   warp 8      TMA producer, both CTAs: loads into its own shared memory,
//               completion bytes counted on CTA 0's full barrier
//   warp 9      CTA 0: block-scale copies and MMAs for the pair
// Synchronisation across the pair:
//   full[s]     CTA 0 only; CTA 0's producer arms it with both CTAs' bytes
//   empty[s]    both CTAs; the MMA warp's commit multicasts to both
//   acc_full    both CTAs; multicast commit after a tile's last MMA
//   acc_empty   CTA 0 only; the 16 epilogue warps of both CTAs arrive on it
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
constexpr int EPI_WARPS = 8;
constexpr int PRODUCER_WARP = 8;
constexpr int MMA_WARP = 9;
constexpr int NUM_THREADS = (MMA_WARP + 1) * 32;
constexpr int EPI_COLS = BN / 2;                  // columns per epilogue warp
constexpr int EPI_CHUNK = 16;                     // columns per TMA store
constexpr int EPI_BUF_BYTES = 32 * EPI_CHUNK * 2;
constexpr int EPI_BYTES = EPI_WARPS * 2 * EPI_BUF_BYTES;
constexpr int TMEM_COLS = 512;
constexpr int SF_COLS = 48;                       // SFA 16 + SFB 32 columns per K slice
constexpr int TMEM_SF0 = BN;                      // scale buffer s at TMEM_SF0 + s * SF_COLS
constexpr int TMEM_SFA_OFF = 0, TMEM_SFB_OFF = 16;
static_assert(TMEM_SF0 + STAGES * SF_COLS <= TMEM_COLS, "one scale buffer per stage above the accumulator");
constexpr uint16_t PAIR_MASK = 0x3;
constexpr unsigned long long kDrainLimitNs = 2000000000ull;

struct SmemCtl {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t acc_full;
  uint64_t acc_empty;
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

constexpr size_t SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + EPI_BYTES + sizeof(SmemCtl);
static_assert(SMEM_BYTES <= 232448, "fits the 227 KB opt-in shared memory of one CTA");

// Instruction descriptors for M = 256 (the pair), N = 256.
constexpr uint32_t IDESC_NVFP4 = (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(256 >> 4) << 24);
constexpr uint32_t IDESC_BF16 =
    (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(256 >> 4) << 24);

SVDQ_DEV uint64_t sw128_desc(uint32_t saddr) { return smem_desc(saddr, 16, 1024, 2); }
SVDQ_DEV uint64_t sf_desc(uint32_t saddr) { return smem_desc(saddr, 0, 128, 0); }

// bf16 pair (low half = the even column) -> two floats.
SVDQ_DEV float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
SVDQ_DEV float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

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
  const int slices = k_tiles + 1;  // + the low-rank slice (slice 0, no block scales)

  // Every CTA initialises the same barrier set; only CTA 0's full[],
  // acc_empty and drain barriers are used.
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&ctl->full[s]), 1);
      mbar_init(smem_u32(&ctl->empty[s]), 1);
    }
    mbar_init(smem_u32(&ctl->acc_full), 1);
    mbar_init(smem_u32(&ctl->acc_empty), 2 * EPI_WARPS);
    mbar_init(smem_u32(&ctl->drain), 1);
    ctl->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == PRODUCER_WARP && lane == 0) {
    prefetch_tmap(&tm_a);
    prefetch_tmap(&tm_b);
    prefetch_tmap(&tm_la);
    prefetch_tmap(&tm_lb);
    prefetch_tmap(&tm_y);
    prefetch_tmap(&tm_sfa);
    prefetch_tmap(&tm_sfb);
  }
  if (warp == MMA_WARP) {
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

  if (warp == PRODUCER_WARP) {
    {
      // ------------------------------------------------------------ producer
      // The whole warp runs the loop; one elected lane issues the copies.
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
          if (!mbar_wait_warp(smem_u32(&ctl->empty[stage]), phase ^ 1, wctx, kDevTimeoutProducer)) {
            ok = false;
            break;
          }
          uint8_t* sa = stage_base + stage * STAGE_BYTES;
          uint8_t* sb = sa + A_BYTES;
          uint8_t* ssfa = sb + B_BYTES;
          uint8_t* ssfb = ssfa + SFA_BYTES;
          const uint32_t full_local = smem_u32(&ctl->full[stage]);
          const uint32_t full = rank == 0 ? full_local : mapa_shared(full_local, 0);
          if (!elect_one()) {
          } else if (kt == 0) {
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
          __syncwarp();
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
  } else if (warp == MMA_WARP) {
    if (rank == 0) {
      // ------------------------------------------------------------ MMA issuer (CTA 0)
      // The whole warp runs the loop; the same elected lane (the lowest)
      // issues every MMA and commit, since a commit tracks the MMAs of the
      // thread that issues it.
      int stage = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int tile = pair; tile < num_tiles && ok; tile += num_pairs) {
        // Both CTAs' epilogues have taken the previous tile's accumulator.
        if (!mbar_wait_warp(smem_u32(&ctl->acc_empty), acc_phase ^ 1, wctx, kDevTimeoutMma)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int kt = 0; kt < slices; ++kt) {
          if (!mbar_wait_warp(smem_u32(&ctl->full[stage]), phase, wctx, kDevTimeoutMma)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(stage_base + stage * STAGE_BYTES);
          const uint32_t sb = sa + A_BYTES;
          const bool leader = elect_one();
          if (!leader) {
          } else if (kt == 0) {
#pragma unroll
            for (int j = 0; j < 4; ++j)
              mma_bf16_pair(tmem, sw128_desc(sa + 32 * j), sw128_desc(sb + 32 * j), IDESC_BF16, j > 0 ? 1u : 0u);
          } else {
            // Scales smem -> this stage's TMEM buffer in both CTAs: per K64
            // chunk j, SFA (4 columns) and the SFB of the tile's two 128-row
            // blocks (4 columns each).
            const uint32_t sf = tmem + TMEM_SF0 + stage * SF_COLS;
            const uint32_t ssf = sa + A_BYTES + B_BYTES;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              tmem_cp_pair_32x128_warpx4(sf + TMEM_SFA_OFF + 4 * j, sf_desc(ssf + 512 * j));
              tmem_cp_pair_32x128_warpx4(sf + TMEM_SFB_OFF + 8 * j, sf_desc(ssf + SFA_BYTES + 512 * j));
              tmem_cp_pair_32x128_warpx4(sf + TMEM_SFB_OFF + 4 + 8 * j, sf_desc(ssf + 2 * SFA_BYTES + 512 * j));
            }
#pragma unroll
            for (int j = 0; j < 4; ++j)
              mma_nvfp4_pair(tmem, sw128_desc(sa + 32 * j), sw128_desc(sb + 32 * j), IDESC_NVFP4,
                             sf + TMEM_SFA_OFF + 4 * j, sf + TMEM_SFB_OFF + 8 * j, 1u);
          }
          // Both CTAs may refill this stage (and its scale buffer) once the
          // copies and MMAs reading it are done.
          if (leader) tc_commit_pair_mc(smem_u32(&ctl->empty[stage]), PAIR_MASK);
          __syncwarp();
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        if (elect_one()) tc_commit_pair_mc(smem_u32(&ctl->acc_full), PAIR_MASK);
        __syncwarp();
        acc_phase ^= 1;
      }
      // Wait for every MMA the elected lane issued before tensor memory is freed.
      if (elect_one()) tc_commit_pair(smem_u32(&ctl->drain));
      __syncwarp();
      volatile int never = 0;
      WaitCtx drain_ctx{&never, p.dev_status, kDrainLimitNs};
      mbar_wait(smem_u32(&ctl->drain), 0, drain_ctx, kDevTimeoutDrain);
    }
  } else {
    // -------------------------------------------------------------- epilogue (both CTAs)
    // Warp w owns 32 rows (TMEM lane quarter w % 4) x 128 columns (half
    // w / 4) of this CTA's 128 x 256 accumulator.  It loads all of them with
    // four TMEM loads and one wait, releases the accumulator on CTA 0's
    // acc_empty (remote for CTA 1), and only then converts and stores.
    const int q = warp & 3, h = warp >> 2;
    uint8_t* buf0 = epi_base + warp * 2 * EPI_BUF_BYTES;
    const uint32_t acc_empty_local = smem_u32(&ctl->acc_empty);
    const uint32_t acc_empty_leader = rank == 0 ? acc_empty_local : mapa_shared(acc_empty_local, 0);
    const uint32_t acc_base = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(h * EPI_COLS);
    uint32_t acc_phase = 0;
    int chunk_seq = 0;
    for (int tile = pair; tile < num_tiles; tile += num_pairs) {
      const int m0 = (tile % tiles_m) * 2 * BM + (int)rank * BM;
      const int nw = (tile / tiles_m) * BN + h * EPI_COLS;   // this warp's first column
      // Lane l holds the bias of columns nw + 4 l .. nw + 4 l + 3.
      uint2 bias4 = make_uint2(0, 0);
      if (p.bias != nullptr && nw + 4 * lane < p.N) bias4 = __ldg(reinterpret_cast<const uint2*>(p.bias + nw) + lane);
      const bool got = mbar_wait(smem_u32(&ctl->acc_full), acc_phase, wctx, kDevTimeoutEpilogue);
      if (!__all_sync(0xffffffffu, got)) break;  // warp-uniform decision
      tc_fence_after();
      uint32_t r[4][32];
#pragma unroll
      for (int i = 0; i < 4; ++i) tmem_ld_32x32b_x32(acc_base + 32 * i, r[i]);
      tmem_ld_wait(r[0]);
      reg_fence(r[1]);
      reg_fence(r[2]);
      reg_fence(r[3]);
      // The loads are complete (wait::ld) and ordered before the arrive by
      // the tcgen05 fence, which is all the MMA warp needs before it
      // overwrites the accumulator: CTA 1's remote arrive is relaxed.
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (rank == 0)
          mbar_arrive(acc_empty_local);
        else
          mbar_arrive_cluster_relaxed(acc_empty_leader);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {      // two 16-column halves per TMEM load
          const int c0 = 32 * i + EPI_CHUNK * hh;
          const int ncol = nw + c0;
          uint32_t bw[8];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            bw[2 * j] = __shfl_sync(0xffffffffu, bias4.x, c0 / 4 + j);
            bw[2 * j + 1] = __shfl_sync(0xffffffffu, bias4.y, c0 / 4 + j);
          }
          uint32_t packed[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const float y0 = __fmaf_rn(p.alpha, __uint_as_float(r[i][hh * 16 + 2 * k]), bf16_lo(bw[k]));
            const float y1 = __fmaf_rn(p.alpha, __uint_as_float(r[i][hh * 16 + 2 * k + 1]), bf16_hi(bw[k]));
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
  if (warp == MMA_WARP) {
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
