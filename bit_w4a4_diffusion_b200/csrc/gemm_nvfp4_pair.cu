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
// Roles (10 warps per CTA, 12 with a fused epilogue; the MMA warp is idle in
// CTA 1):
//   warps 0..7  epilogue, both CTAs: warp w reads TMEM lane quarter w % 4,
//               columns [128 (w / 4), + 128) of the tile
//   warp 8      TMA producer, both CTAs: loads into its own shared memory,
//               completion bytes counted on CTA 0's full barrier
//   warp 9      CTA 0: block-scale copies and MMAs for the pair
//   warps 10,11 fused epilogues only: idle (they complete the third
//               warpgroup, which hands registers to the epilogue warpgroups
//               with setmaxnreg)
// Epilogues: y = bf16(alpha D + b) through TMA stores; the GELU-MLP
// epilogue (GELU, the down layer's NVFP4 quantizer and its low-rank
// down-projection partials); the QKV epilogue (RMSNorm of the Q and K heads
// and RoPE).  The fused ones are those of the single-CTA kernel
// (gemm_nvfp4.cu), reading the whole 128-column accumulator slice of a warp
// before releasing it.
// Synchronisation across the pair:
//   full[s]     CTA 0 only; CTA 0's producer arms it with both CTAs' bytes
//   empty[s]    both CTAs; the MMA warp's commit multicasts to both
//   acc_full    both CTAs; multicast commit after a tile's last MMA
//   acc_empty   CTA 0 only; the 16 epilogue warps of both CTAs arrive on it
// Every mbarrier wait is bounded; on timeout the kernel records a status code,
// drains what it can observe, and both CTAs meet at the final cluster barrier.
//
// The same pipeline also runs the INT4 layer's product on fp16 operands
// (EPI_F16; the operands come from dequant_int4.cu, exact fp16 values of the
// dequantized codes, each row scaled by a power of two): the K slices are 64
// fp16 elements (128 bytes, one 64-group) with four kind::f16 MMAs each and
// no block scales, the low-rank slice is the same, and the epilogue applies
// the rows' and columns' powers of two: y = bf16(D f_a[m] f_w[n] + bias).
#include <cuda_bf16.h>
#include <cstdint>

#include "epilogue.cuh"
#include "fused_quant.cuh"
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
constexpr int EPI_PLAIN = 0, EPI_GELU = 1, EPI_QKV = 2, EPI_F16 = 3;
template <int kEpi>
constexpr bool fused_epi() { return kEpi == EPI_GELU || kEpi == EPI_QKV; }
template <int kEpi>
constexpr int num_threads() { return fused_epi<kEpi>() ? 12 * 32 : (MMA_WARP + 1) * 32; }
// Fused epilogues: launched at 168 registers per thread; the third warpgroup
// (producer, MMA, two idle warps) drops to 72 and the two epilogue
// warpgroups rise to 216.
constexpr int FUSED_LAUNCH_REGS = 168, FUSED_EPI_REGS = 216, FUSED_CTL_REGS = 72;
static_assert(256 * FUSED_EPI_REGS + 128 * FUSED_CTL_REGS <= 384 * FUSED_LAUNCH_REGS, "register split");
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
  int unit;        // fused layer kernel: the quantizer unit the epilogue warps took
  int last;        // ... and whether it was the last unit of its row block
  uint64_t qfull[2];   // fused layer kernel: a quantizer chunk landed in buffer b
};

// The fused epilogues keep per-tile column tables after the staging area:
// GELU 1/lambda (fp32) + bias (bf16), QKV gamma_q | gamma_k (fp32) + bias;
// the fused layer kernel keeps its quantizer's 1/d table (256 fp32) there.
constexpr int TABLE_BYTES = BN * 4 + BN * 2;
static_assert(TABLE_BYTES >= 256 * 4, "room for the quantizer's reciprocal table");
// The fused layer kernel keeps 4 GEMM stages and gives the fifth's room to
// the quantizer's two chunk buffers (fused_quant.cuh).
template <bool kQuant>
constexpr int stages() { return kQuant ? 4 : STAGES; }
template <int kEpi, bool kQuant>
constexpr size_t smem_bytes() {
  return 1024 + stages<kQuant>() * STAGE_BYTES + EPI_BYTES + (kQuant ? 2 * QC_BUF_BYTES : 0) +
         (fused_epi<kEpi>() || kQuant ? TABLE_BYTES : 0) + sizeof(SmemCtl);
}
static_assert(QC_BUF_BYTES % 1024 == 0 && EPI_BYTES % 1024 == 0, "chunk buffers keep the SWIZZLE_128B alignment");
static_assert(smem_bytes<EPI_GELU, false>() <= 232448, "fits the 227 KB opt-in shared memory of one CTA");
static_assert(smem_bytes<EPI_PLAIN, true>() <= 232448, "fits the 227 KB opt-in shared memory of one CTA");

// Instruction descriptors for M = 256 (the pair), N = 256.
constexpr uint32_t IDESC_NVFP4 = (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(256 >> 4) << 24);
constexpr uint32_t IDESC_BF16 =
    (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(256 >> 4) << 24);
// kind::f16 with fp16 A and B (format 0), fp32 D.
constexpr uint32_t IDESC_F16 = (1u << 4) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(256 >> 4) << 24);

SVDQ_DEV uint64_t sw128_desc(uint32_t saddr) { return smem_desc(saddr, 16, 1024, 2); }
SVDQ_DEV uint64_t sf_desc(uint32_t saddr) { return smem_desc(saddr, 0, 128, 0); }

// bf16 pair (low half = the even column) -> two floats.
SVDQ_DEV float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
SVDQ_DEV float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

template <int kEpi, bool kQuant>
__global__ void __launch_bounds__(num_threads<kEpi>(), 1)
    gemm_nvfp4_pair_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                           const __grid_constant__ CUtensorMap tm_la, const __grid_constant__ CUtensorMap tm_lb,
                           const __grid_constant__ CUtensorMap tm_y, const __grid_constant__ CUtensorMap tm_sfa,
                           const __grid_constant__ CUtensorMap tm_sfb, const __grid_constant__ CUtensorMap tm_x,
                           const __grid_constant__ CUtensorMap tm_l1, const GemmNvfp4Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  constexpr int kStages = stages<kQuant>();
  uint8_t* stage_base = smem;
  uint8_t* epi_base = smem + kStages * STAGE_BYTES;
  constexpr bool kGelu = kEpi == EPI_GELU, kFused = fused_epi<kEpi>();
  constexpr bool kF16 = kEpi == EPI_F16;
  static_assert(kEpi >= EPI_PLAIN && kEpi <= EPI_F16, "epilogue kind");
  static_assert(!kQuant || kEpi == EPI_PLAIN, "the fused layer kernel has the plain epilogue");
  // Fused layer kernel: the quantizer's chunk buffers, then its 1/d table.
  uint8_t* q_base = epi_base + EPI_BYTES;
  uint8_t* table_base = q_base + (kQuant ? 2 * QC_BUF_BYTES : 0);
  SmemCtl* ctl = reinterpret_cast<SmemCtl*>(table_base + (kFused || kQuant ? TABLE_BYTES : 0));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();     // 0: leader (issues the MMAs), 1: peer
  const int pair = blockIdx.x >> 1, num_pairs = gridDim.x >> 1;
  const int tiles_m = (p.M + 2 * BM - 1) / (2 * BM);
  const int tiles_n = (p.N + BN - 1) / BN;
  const int num_tiles = tiles_m * tiles_n;
  const int k_tiles = kF16 ? p.K / 64 : p.K / 256;
  const int slices = k_tiles + 1;  // + the low-rank slice (slice 0, no block scales)
  // Tile schedule.  Plain and QKV epilogues: round robin over tiles numbered
  // M-block fastest.  GELU-MLP epilogue: cluster i takes the contiguous run
  // [i T / G, (i + 1) T / G) of tiles numbered N-block fastest, so that its
  // consecutive tiles share an M-block and the epilogue can carry the
  // low-rank partial of those rows from tile to tile.
  // Fused layer kernel: round robin over tiles numbered N-block fastest, so
  // that the first wave needs only the first M-blocks of x quantized.
  constexpr bool kNFast = kGelu || kQuant;
  const int t_begin = kGelu ? (int)((long long)pair * num_tiles / num_pairs) : pair;
  const int t_end = kGelu ? (int)((long long)(pair + 1) * num_tiles / num_pairs) : num_tiles;
  const int t_step = kGelu ? 1 : num_pairs;
  auto tile_m0 = [&](int tile) { return (kNFast ? tile / tiles_n : tile % tiles_m) * 2 * BM + (int)rank * BM; };
  auto tile_n0 = [&](int tile) { return (kNFast ? tile % tiles_n : tile / tiles_m) * BN; };
  float* rcp_tab = reinterpret_cast<float*>(table_base);   // fused layer kernel only
  if constexpr (kQuant) {
    // The reciprocal each group's codes are scaled by, for every scale byte
    // the quantizer can produce (0 marks an all-zero group), as in the
    // quantize kernel.
    if (threadIdx.x < 256) {
      const float d = __fmul_rn(e4m3_to_f32(threadIdx.x), p.fq.act_scale);
      rcp_tab[threadIdx.x] = d != 0.f ? __frcp_rn(d) : 0.f;
    }
  }

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
    mbar_init(smem_u32(&ctl->qfull[0]), 1);
    mbar_init(smem_u32(&ctl->qfull[1]), 1);
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

  // Inputs produced by the preceding kernel become visible here.
  pdl_wait();
  // The next kernel on the stream may be scheduled from now on; it waits for
  // this grid's completion before it reads anything.
  pdl_launch_dependents();

  WaitCtx wctx{&ctl->abort_flag, p.dev_status, p.timeout_ns};
  const int total_units = kQuant ? p.fq.row_blocks * p.fq.splits : 0;
  if constexpr (kQuant) {
    // (No L2 prefetch of x: issued at kernel entry it competes for HBM with
    // the first units' own chunk loads, which decide when the GEMM starts.)
    if (threadIdx.x == 0) {
      prefetch_tmap(&tm_x);
      prefetch_tmap(&tm_l1);
    }
  }

  // ---------------------------------------------------------------- roles
  auto role_producer = [&]() {
    {
      // ------------------------------------------------------------ producer
      // The whole warp runs the loop; one elected lane issues the copies.
      // Loads of a K slice split into the weight side (B codes and scales, or
      // [L2^T|L2^T] for the low-rank slice) and the activation side (A codes
      // and scales, or lora_act).  In the fused layer kernel the activation
      // side of a 128-row block exists only once the block's ready word is
      // set: at the first tile of a new row block the producer issues the
      // weight side of up to kStages slices, waits for the word, then issues
      // their activation side.
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_phase = 0;  // CTA 0: per stage, load outstanding and its parity
      bool ok = true;
      const uint64_t pol = policy_evict_last();   // every operand is re-read by other tiles
      const int kch = p.K / 64;
      // Fused layer kernel: the last row block seen ready, and the ready word
      // of the next tile's row block, read (acquire) one tile ahead so that
      // its latency hides behind the filled ring.
      int ready_rb = -1, ahead_rb = -1, ahead_val = 0;
      auto stage_ptr = [&](int st) { return stage_base + st * STAGE_BYTES; };
      auto full_addr = [&](int st) {
        const uint32_t local = smem_u32(&ctl->full[st]);
        return rank == 0 ? local : mapa_shared(local, 0);
      };
      auto issue_weight = [&](int st, int kt, int n0, int nb) {
        uint8_t* sa = stage_ptr(st);
        uint8_t* sb = sa + A_BYTES;
        uint8_t* ssfb = sb + B_BYTES + SFA_BYTES;
        const uint32_t full = full_addr(st);
        if (rank == 0) mbar_arrive_expect_tx(smem_u32(&ctl->full[st]), kt == 0 || kF16 ? 2 * (A_BYTES + B_BYTES)
                                                                                      : 2 * STAGE_BYTES);
        if (kt == 0) {
          tma_load_2d_pair(smem_u32(sb), &tm_lb, 0, nb, full, pol);
        } else if (kF16) {
          tma_load_2d_pair(smem_u32(sb), &tm_b, (kt - 1) * BK_BYTES, nb, full, pol);
        } else {
          const int kb = kt - 1;
          tma_load_2d_pair(smem_u32(sb), &tm_b, kb * BK_BYTES, nb, full, pol);
          // Scales: 256-byte rows of the tiled layout, 2 KB (8 rows) per
          // 128-row block and K slice.
          tma_load_2d_pair(smem_u32(ssfb), &tm_sfb, 0, ((n0 / 128) * kch + kb * 4) * 2, full, pol);
          tma_load_2d_pair(smem_u32(ssfb + SFA_BYTES), &tm_sfb, 0, ((n0 / 128 + 1) * kch + kb * 4) * 2, full, pol);
        }
      };
      auto issue_act = [&](int st, int kt, int m0) {
        uint8_t* sa = stage_ptr(st);
        uint8_t* ssfa = sa + A_BYTES + B_BYTES;
        const uint32_t full = full_addr(st);
        if (kt == 0) {
          tma_load_2d_pair(smem_u32(sa), &tm_la, 0, m0, full, pol);
        } else {
          const int kb = kt - 1;
          tma_load_2d_pair(smem_u32(sa), &tm_a, kb * BK_BYTES, m0, full, pol);
          if (!kF16) tma_load_2d_pair(smem_u32(ssfa), &tm_sfa, 0, ((m0 / 128) * kch + kb * 4) * 2, full, pol);
        }
      };
      auto advance = [&]() {
        issued_mask |= 1u << stage;
        issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1;
        }
      };
      for (int tile = t_begin; tile < t_end && ok; tile += t_step) {
        const int m0 = tile_m0(tile);                                  // this CTA's A rows
        const int n0 = tile_n0(tile);                                  // the tile's B rows
        const int nb = n0 + (int)rank * BN_HALF;                       // this CTA's half of them
        int kt0 = 0;
        if (kQuant && (m0 >> 7) != ready_rb) {
          const int rb = m0 >> 7;
          int v = (rb == ahead_rb) ? ahead_val : 0;
          if (v == 0) {
            if (lane == 0) v = ld_acquire_gpu(p.fq.sync + kSyncReady + rb);
            v = __shfl_sync(0xffffffffu, v, 0);
          }
          if (v != 0) {
            // The rows were written through the generic proxy by other SMs;
            // the TMA reads them through the async proxy.
            fence_proxy_async_global();
            ready_rb = rb;
          }
        }
        if (kQuant && tile + t_step < t_end) {
          const int nrb = tile_m0(tile + t_step) >> 7;
          if (nrb != ahead_rb && nrb != ready_rb) {
            int v = 0;
            if (lane == 0) v = ld_acquire_gpu(p.fq.sync + kSyncReady + nrb);
            ahead_val = __shfl_sync(0xffffffffu, v, 0);
            ahead_rb = nrb;
          }
        }
        if (kQuant && (m0 >> 7) != ready_rb) {
          // Not ready yet: the weight side of the first slices, then the wait.
          const int rb = m0 >> 7;
          const int P = slices < kStages ? slices : kStages;
          const int st0 = stage;
          for (int kt = 0; kt < P; ++kt) {
            if (!mbar_wait_warp(smem_u32(&ctl->empty[stage]), phase ^ 1, wctx, kDevTimeoutProducer)) {
              ok = false;
              break;
            }
            if (elect_one()) issue_weight(stage, kt, n0, nb);
            __syncwarp();
            advance();
          }
          if (!ok) {
            // The weight side of the stages issued so far is in flight; their
            // barriers complete only with the activation side, which the
            // drain below does not wait for: give it the (possibly stale)
            // rows so that every armed stage completes.
            kt0 = -1;
          } else {
            bool got = true;
            if (lane == 0) got = flag_wait(p.fq.sync + kSyncReady + rb, wctx, kDevTimeoutProducer);
            got = __shfl_sync(0xffffffffu, got, 0) != 0;
            // The rows were written through the generic proxy by other SMs;
            // the TMA reads them through the async proxy.
            fence_proxy_async_global();
            if (!got) ok = false;
            ready_rb = got ? rb : ready_rb;
            kt0 = P;
          }
          // Activation side of the stages just armed (also after a timeout,
          // so that no armed barrier is left without its bytes).
          const int armed = kt0 < 0 ? (stage - st0 + kStages) % kStages : P;   // < kStages when the loop broke
          if (elect_one())
            for (int i = 0; i < armed; ++i) issue_act((st0 + i) % kStages, i, m0);
          __syncwarp();
          if (!ok) break;
        }
        for (int kt = kt0; kt < slices; ++kt) {
          if (!mbar_wait_warp(smem_u32(&ctl->empty[stage]), phase ^ 1, wctx, kDevTimeoutProducer)) {
            ok = false;
            break;
          }
          if (elect_one()) {
            issue_weight(stage, kt, n0, nb);
            issue_act(stage, kt, m0);
          }
          __syncwarp();
          advance();
        }
      }
      // CTA 0 never leaves with copies in flight into the pair's shared
      // memory: a full[] phase completes only when both CTAs' bytes landed.
      if (rank == 0) {
        volatile int never = 0;
        WaitCtx drain_ctx{&never, p.dev_status, kDrainLimitNs};
        for (int s = 0; s < kStages; ++s)
          if (issued_mask & (1u << s))
            mbar_wait(smem_u32(&ctl->full[s]), (issued_phase >> s) & 1, drain_ctx, kDevTimeoutDrain);
      }
    }
  };
  auto role_mma = [&]() {
    if (rank == 0) {
      // ------------------------------------------------------------ MMA issuer (CTA 0)
      // The whole warp runs the loop; the same elected lane (the lowest)
      // issues every MMA and commit, since a commit tracks the MMAs of the
      // thread that issues it.
      int stage = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int tile = t_begin; tile < t_end && ok; tile += t_step) {
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
          } else if (kF16) {
            // 64 fp16 elements: four K = 16 steps of 32 bytes in the swizzled rows.
#pragma unroll
            for (int j = 0; j < 4; ++j)
              mma_bf16_pair(tmem, sw128_desc(sa + 32 * j), sw128_desc(sb + 32 * j), IDESC_F16, 1u);
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
          if (++stage == kStages) {
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
  };
  auto role_epilogue_plain = [&]() {
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
    // Fused layer kernel: quantizer units (fused_quant.cuh) while this CTA's
    // accumulator is not ready (until_acc) or until the queue is empty.  All
    // eight warps take every decision together (named barriers 2 and 3), so
    // that they work on one unit at a time and stay in step.  A unit's
    // 64-column chunks come through the two TMA-fed buffers: thread 0 issues
    // the first two when it takes the unit and chunk c + 2 once every warp is
    // done with chunk c.  A CTA's first unit is unit blockIdx.x, known without
    // the queue, so that its loads start at kernel entry; the queue hands out
    // units from gridDim.x on.
    constexpr int NT = EPI_WARPS * 32;
    bool units_left = kQuant;
    const int span = p.K / (kQuant ? p.fq.splits : 1), nch = span / QC_COLS;
    uint32_t qseq = 0;                       // chunk loads issued by this CTA so far (uniform)
    uint32_t q_issued_mask = 0, q_issued_phase = 0;   // thread 0: last load per buffer, for the drain
    const uint32_t qb0 = smem_u32(q_base);
    auto issue_chunk = [&](int rb, int k, uint32_t seq) {   // thread 0
      const int b = (int)(seq & 1);
      const uint32_t buf = qb0 + (uint32_t)b * QC_BUF_BYTES;
      const uint32_t bar = smem_u32(&ctl->qfull[b]);
      fence_proxy_async_smem();   // the buffer's generic reads (chunk seq - 2) before the async-proxy writes
      mbar_arrive_expect_tx(bar, QC_TX_BYTES);
      tma_load_2d(buf, &tm_x, k, rb * 128, bar);
      tma_load_2d(buf + QC_X_BYTES, &tm_l1, k, 0, bar);
      bulk_load(buf + QC_X_BYTES + QC_L_BYTES, p.fq.inv_smooth + k, QC_I_BYTES, bar);
      q_issued_mask |= 1u << b;
      q_issued_phase = (q_issued_phase & ~(1u << b)) | (((seq >> 1) & 1) << b);
    };
    const float q_inv_six_s = kQuant ? __frcp_rn(__fmul_rn(6.0f, p.fq.act_scale)) : 0.f;
    const float2 q_xs2 = make_float2(p.fq.lr_in_scale, p.fq.lr_in_scale);
    auto issue_first_chunks = [&](int u) {   // thread 0
      if (u < total_units) {
        const int rb = u / p.fq.splits, k0 = (u - rb * p.fq.splits) * span;
        issue_chunk(rb, k0, qseq);
        if (nch > 1) issue_chunk(rb, k0 + QC_COLS, qseq + 1);
      }
    };
    bool first_unit = kQuant;
    if (kQuant && threadIdx.x == 0) {
      ctl->unit = (int)blockIdx.x;
      issue_first_chunks((int)blockIdx.x);
    }
    auto run_units = [&](bool until_acc) {
      while (units_left) {
        const bool stop = until_acc && mbar_test_wait(smem_u32(&ctl->acc_full), acc_phase);
        if (named_bar_any(2, NT, stop || *reinterpret_cast<volatile int*>(&ctl->abort_flag) != 0)) return;
        if (threadIdx.x == 0 && !first_unit) {
          const int u = atomicAdd(p.fq.sync + kSyncQueue, 1) + (int)gridDim.x;
          ctl->unit = u;
          issue_first_chunks(u);
        }
        first_unit = false;
        named_bar_sync(3, NT);
        const int u = ctl->unit;
        if (u >= total_units) {
          units_left = false;
          return;
        }
        const int rb = u / p.fq.splits, sp = u - rb * p.fq.splits, k0 = sp * span;
        // The lane's rows within the unit: 16 w + perm(g), + 8.
        const int g = lane >> 2, c = lane & 3;
        const int r0 = 16 * warp + quant_perm(g);
        QuantLane L;
        L.row0 = rb * 128 + r0;
        L.K = p.K;
        L.c = c;
        L.ok0 = L.row0 < p.M;
        L.ok1 = L.row0 + 8 < p.M;
        L.code0 = p.fq.codes + (size_t)L.row0 * (p.K / 2) + 4 * c;
        L.xr0 = nullptr;
        L.inv = nullptr;
        L.l1t = nullptr;
        float qacc[4][4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
          for (int e = 0; e < 4; ++e) qacc[j][e] = 0.f;
        bool ok = true;
        for (int ch = 0; ch < nch; ++ch) {
          const uint32_t seq = qseq + ch;
          const int b = (int)(seq & 1);
          const bool got = mbar_wait(smem_u32(&ctl->qfull[b]), (seq >> 1) & 1, wctx, kDevTimeoutEpilogue);
          if (named_bar_any(3, NT, !got)) {
            ok = false;
            break;
          }
          quant_chunk(qb0 + (uint32_t)b * QC_BUF_BYTES, k0 + QC_COLS * ch, L, r0, rcp_tab, q_inv_six_s, q_xs2,
                      p.fq.scales, qacc);
          named_bar_sync(3, NT);   // every warp is done with buffer b
          if (threadIdx.x == 0 && ch + 2 < nch) issue_chunk(rb, k0 + QC_COLS * (ch + 2), seq + 2);
        }
        if (!ok) {
          units_left = false;
          return;
        }
        qseq += nch;
        // The warp's low-rank partial: row r0 (r0 + 8), ranks 8 j + c and 8 j + 4 + c.
        {
          const size_t mp = (size_t)p.fq.row_blocks * 128;
          float* u0 = p.fq.u_part + ((size_t)sp * mp + L.row0) * 32 + c;
          float* u1 = u0 + 8 * 32;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            __stcg(u0 + 8 * j, qacc[j][0]);
            __stcg(u0 + 8 * j + 4, qacc[j][1]);
            __stcg(u1 + 8 * j, qacc[j][2]);
            __stcg(u1 + 8 * j + 4, qacc[j][3]);
          }
        }
        // Publish the unit: the barrier orders every thread's stores before
        // thread 0's fence and count (one count per unit).
        named_bar_sync(3, NT);
        if (threadIdx.x == 0)
          ctl->last = atomic_add_acq_rel_gpu(p.fq.sync + kSyncCount + rb, 1) == p.fq.splits - 1;
        named_bar_sync(3, NT);
        if (ctl->last) {
          // The last unit of the block: every other unit's partials are
          // visible (thread 0 saw all counts, then fenced, then the barrier);
          // add them up, then raise the block's ready word.
          reduce_row_block(p.fq, p.M, rb, threadIdx.x);
          named_bar_sync(3, NT);
          if (threadIdx.x == 0) {
            fence_proxy_async_global();
            st_release_gpu(p.fq.sync + kSyncReady + rb, 1);
          }
        }
      }
    };
    for (int tile = t_begin; tile < t_end; tile += t_step) {
      if constexpr (kQuant) run_units(true);
      const int m0 = tile_m0(tile);
      const int nw = tile_n0(tile) + h * EPI_COLS;   // this warp's first column
      // Lane l holds the bias of columns nw + 4 l .. nw + 4 l + 3.
      uint2 bias4 = make_uint2(0, 0);
      if (p.bias != nullptr && nw + 4 * lane < p.N) bias4 = __ldg(reinterpret_cast<const uint2*>(p.bias + nw) + lane);
      // fp16-operand kernel: the row's power of two (this lane's row) and,
      // in lane l, those of columns nw + 4 l .. + 3.
      float f_row = 0.f;
      float4 f_col4 = make_float4(0.f, 0.f, 0.f, 0.f);
      if constexpr (kF16) {
        const int row = m0 + 32 * q + lane;
        if (row < p.M) f_row = __ldg(p.row_factor + row);
        if (nw + 4 * lane < p.N) f_col4 = __ldg(reinterpret_cast<const float4*>(p.col_factor + nw) + lane);
      }
      const bool got = mbar_wait(smem_u32(&ctl->acc_full), acc_phase, wctx, kDevTimeoutEpilogue);
      if constexpr (kQuant) {
        if (named_bar_any(2, NT, !got)) break;   // decided by all eight warps
      } else {
        if (!__all_sync(0xffffffffu, got)) break;  // warp-uniform decision
      }
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
          // Per column, the factor D is multiplied by: alpha, or for the
          // fp16-operand kernel f_a[row] f_w[col] (a power of two, so the
          // fma below still rounds once).
          float fc[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) fc[j] = p.alpha;
          if constexpr (kF16) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              fc[4 * j] = __fmul_rn(f_row, __shfl_sync(0xffffffffu, f_col4.x, c0 / 4 + j));
              fc[4 * j + 1] = __fmul_rn(f_row, __shfl_sync(0xffffffffu, f_col4.y, c0 / 4 + j));
              fc[4 * j + 2] = __fmul_rn(f_row, __shfl_sync(0xffffffffu, f_col4.z, c0 / 4 + j));
              fc[4 * j + 3] = __fmul_rn(f_row, __shfl_sync(0xffffffffu, f_col4.w, c0 / 4 + j));
            }
          }
          uint32_t packed[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const float y0 = __fmaf_rn(fc[2 * k], __uint_as_float(r[i][hh * 16 + 2 * k]), bf16_lo(bw[k]));
            const float y1 = __fmaf_rn(fc[2 * k + 1], __uint_as_float(r[i][hh * 16 + 2 * k + 1]), bf16_hi(bw[k]));
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
    // Units nobody has taken yet (other CTAs' tiles may wait for them).
    if constexpr (kQuant) {
      run_units(false);
      // Never leave with a chunk load in flight into shared memory.
      if (threadIdx.x == 0) {
        volatile int never = 0;
        WaitCtx drain_ctx{&never, p.dev_status, kDrainLimitNs};
        for (int b = 0; b < 2; ++b)
          if (q_issued_mask & (1u << b))
            mbar_wait(smem_u32(&ctl->qfull[b]), (q_issued_phase >> b) & 1, drain_ctx, kDevTimeoutDrain);
      }
    }
    if (lane == 0) bulk_wait<0>();
  };
  // Release of the accumulator by one epilogue warp: CTA 0's warps arrive
  // locally, CTA 1's remotely with relaxed semantics (the TMEM loads are
  // complete and fenced before it).
  auto release_acc = [&]() {
    tc_fence_before();
    __syncwarp();
    if (lane == 0) {
      const uint32_t local = smem_u32(&ctl->acc_empty);
      if (rank == 0)
        mbar_arrive(local);
      else
        mbar_arrive_cluster_relaxed(mapa_shared(local, 0));
    }
  };
  // Loads this warp's 32 rows x 128 columns of the accumulator, one wait.
  auto load_acc = [&](uint32_t (&r)[4][32], int q, int half) {
    const uint32_t acc_base = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(half * EPI_COLS);
#pragma unroll
    for (int i = 0; i < 4; ++i) tmem_ld_32x32b_x32(acc_base + 32 * i, r[i]);
    tmem_ld_wait(r[0]);
    reg_fence(r[1]);
    reg_fence(r[2]);
    reg_fence(r[3]);
  };

  auto role_epilogue_gelu = [&]() {
    // ------------------------------------------------------ GELU-MLP epilogue
    // Warp w: rows 32 (w mod 4) of the CTA's 128, tile columns
    // [128 (w / 4), + 128), four 32-column chunks of gelu_quant_chunk
    // (epilogue.cuh: GELU, the down layer's quantizer, its low-rank
    // partials).  The tile's 1/lambda and bias columns are staged once per
    // tile in shared memory.  Partial sums of consecutive tiles of one
    // M-block stay in registers and go to u_work with vector reductions when
    // the M-block changes (a separate kernel converts them to lora_act after
    // this grid).  The eight warps share named barriers 2 and 3, so every
    // stop decision is taken by all of them.
    constexpr int NT = EPI_WARPS * 32;
    const int q = warp & 3, hf = warp >> 2;
    const int g = lane >> 2, c = lane & 3;
    const int et = threadIdx.x;  // 0..255 over the epilogue warps
    const GeluQuantParams& gq = p.gq;
    const uint32_t hbase = smem_u32(epi_base + warp * 1024);
    float* tab_inv = reinterpret_cast<float*>(table_base);
    uint16_t* tab_bias = reinterpret_cast<uint16_t*>(table_base + BN * 4);
    const float2 lr2 = make_float2(gq.lr_in_scale, gq.lr_in_scale);
    const float2 alpha2 = make_float2(p.alpha, p.alpha);
    const float inv_six_s = __frcp_rn(__fmul_rn(6.0f, gq.s_d));
    const GeluLane L{tab_inv, tab_bias, alpha2, lr2, inv_six_s, hbase, lane, g, c};
    uint32_t acc_phase = 0;
    // The warp's low-rank partial of its 32 rows: rows 16t + g (+8), ranks
    // 8j + 2c (+1).
    float lacc[2][4][4];
    auto zero_lacc = [&]() {
#pragma unroll
      for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
          for (int e = 0; e < 4; ++e) lacc[t][j][e] = 0.f;
    };
    auto flush_lacc = [&](int mb) {
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const int r0 = mb + 32 * q + 16 * t + g;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int col = 8 * j + 2 * c;
          if (r0 < p.M) red_add_f32x2(gq.u_work + (size_t)r0 * 32 + col, lacc[t][j][0], lacc[t][j][1]);
          if (r0 + 8 < p.M) red_add_f32x2(gq.u_work + (size_t)(r0 + 8) * 32 + col, lacc[t][j][2], lacc[t][j][3]);
        }
      }
    };
    zero_lacc();
    int cur_m0 = -1;
    for (int tile = t_begin; tile < t_end; tile += t_step) {
      const int m0 = tile_m0(tile);
      const int n0 = tile_n0(tile);
      const int row = m0 + 32 * q + lane;
      const bool row_ok = row < p.M;
      // This thread's table column, fetched before the wait.
      const float my_inv = __ldg(gq.inv_smooth + n0 + et);
      const uint16_t my_bias = p.bias != nullptr ? __ldg(p.bias + n0 + et) : (uint16_t)0;
      const bool got = mbar_wait(smem_u32(&ctl->acc_full), acc_phase, wctx, kDevTimeoutEpilogue);
      // All epilogue threads decide together; this barrier also ends every
      // read of the previous tile's table.
      if (named_bar_any(2, NT, !got)) break;
      tab_inv[et] = my_inv;
      tab_bias[et] = my_bias;
      asm volatile("bar.sync 3, %0;" ::"n"(NT) : "memory");
      tc_fence_after();
      if (m0 != cur_m0) {
        if (cur_m0 >= 0) flush_lacc(cur_m0);
        zero_lacc();
        cur_m0 = m0;
      }
      uint32_t rb[4][32];
      load_acc(rb, q, hf);
      release_acc();
      acc_phase ^= 1;
#pragma unroll
      for (int ii = 0; ii < 4; ++ii) {
        const int cl = hf * EPI_COLS + 32 * ii;  // column within the tile
        gelu_quant_chunk(rb[ii], L, gq, p.N, cl, n0 + cl, row, row_ok, lacc);
      }
    }
    if (cur_m0 >= 0) flush_lacc(cur_m0);
  };

  auto role_epilogue_qkv = [&]() {
    // ------------------------------------------ QKV + RMSNorm + RoPE epilogue
    // Warp w: rows 32 (w mod 4) of the CTA's 128, head w / 4 of the tile (a
    // 256-column tile holds two 128-feature heads), by qkv_head
    // (epilogue.cuh: bias, RMSNorm and RoPE for Q and K, bf16 out through a
    // 1 KB shared slab per warp).  The gamma vectors (for the whole kernel)
    // and the tile's bias columns sit in shared memory; the rotary tables are
    // pair-major ([64][M]), so that the 32 rows of a warp read one line per
    // pair.
    constexpr int NT = EPI_WARPS * 32;
    const int q = warp & 3, hf = warp >> 2;
    const int et = threadIdx.x;  // 0..255 over the epilogue warps
    const QkvParams& qp = p.qk;
    const float2 alpha2 = make_float2(p.alpha, p.alpha);
    float* tab_g = reinterpret_cast<float*>(table_base);                  // gamma_q | gamma_k
    uint16_t* tab_bias = reinterpret_cast<uint16_t*>(table_base + 1024);  // 256 bf16
    const uint32_t slab = smem_u32(epi_base + warp * 1024);
    tab_g[et] = et < 128 ? __ldg(qp.gamma_q + et) : __ldg(qp.gamma_k + et - 128);
    uint32_t acc_phase = 0;
    for (int tile = t_begin; tile < t_end; tile += t_step) {
      const int m0 = tile_m0(tile);
      const int n0 = tile_n0(tile);
      const int row = m0 + 32 * q + lane;
      const bool row_ok = row < p.M;
      const int n = n0 + EPI_COLS * hf;  // first column of this warp's head
      const bool head_ok = n < p.N;
      const uint16_t my_bias = (p.bias != nullptr && n0 + et < p.N) ? __ldg(p.bias + n0 + et) : (uint16_t)0;
      const bool got = mbar_wait(smem_u32(&ctl->acc_full), acc_phase, wctx, kDevTimeoutEpilogue);
      // All epilogue threads decide together; this barrier also ends every
      // read of the previous tile's bias columns.
      if (named_bar_any(2, NT, !got)) break;
      tab_bias[et] = my_bias;
      asm volatile("bar.sync 3, %0;" ::"n"(NT) : "memory");
      tc_fence_after();
      uint32_t r[4][32];
      load_acc(r, q, hf);
      release_acc();
      acc_phase ^= 1;
      if (!head_ok) continue;
      const int part = n / qp.hd;  // 0: Q, 1: K, 2: V
      qkv_head(r, tab_bias + EPI_COLS * hf, tab_g + 128 * (part < 2 ? part : 0), alpha2, qp, part, p.M, p.N, row,
               row_ok, m0 + 32 * q, n, slab, lane);
    }
  };

  if constexpr (kFused) {
    // setmaxnreg is warpgroup-wide: the third warpgroup (producer, MMA and
    // two idle warps) gives registers to the two epilogue warpgroups.
    if (warp >= EPI_WARPS) {
      asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(FUSED_CTL_REGS));
      if (warp == PRODUCER_WARP)
        role_producer();
      else if (warp == MMA_WARP)
        role_mma();
    } else {
      asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(FUSED_EPI_REGS));
      if constexpr (kGelu)
        role_epilogue_gelu();
      else
        role_epilogue_qkv();
    }
  } else {
    if (warp == PRODUCER_WARP)
      role_producer();
    else if (warp == MMA_WARP)
      role_mma();
    else
      role_epilogue_plain();
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
  if constexpr (kQuant) {
    // Every role of this CTA is done with the control words.  The last CTA
    // to get here returns them to zero for the next call on this workspace
    // (the next kernel on the stream reads them only after this grid ends).
    if (threadIdx.x == 0) {
      __threadfence();
      if (atomicAdd(p.fq.sync + kSyncExit, 1) == (int)gridDim.x - 1) {
        __threadfence();
        int* sy = p.fq.sync;
        sy[kSyncQueue] = 0;
        sy[kSyncExit] = 0;
        for (int rb = 0; rb < p.fq.row_blocks; ++rb) {
          sy[kSyncCount + rb] = 0;
          sy[kSyncReady + rb] = 0;
        }
        __threadfence();
      }
    }
  }
}

}  // namespace

namespace {
template <int kEpi, bool kQuant>
cudaError_t launch_pair_impl(const GemmNvfp4Params& p, const GemmPairTmaps& t, const CUtensorMap& tm_x,
                             const CUtensorMap& tm_l1, cudaStream_t stream, bool pdl) {
  static int max_pairs = -1;
  auto kernel = gemm_nvfp4_pair_kernel<kEpi, kQuant>;
  constexpr size_t smem = smem_bytes<kEpi, kQuant>();
  if (max_pairs < 0) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if (fused_epi<kEpi>()) {
      // The epilogue warpgroups' setmaxnreg.inc waits until the third
      // warpgroup has released enough registers: only launch if the compiled
      // register count makes the split add up.
      cudaFuncAttributes fa;
      e = cudaFuncGetAttributes(&fa, kernel);
      if (e != cudaSuccess) return e;
      if (fa.numRegs * num_threads<kEpi>() < 256 * FUSED_EPI_REGS + 128 * FUSED_CTL_REGS)
        return cudaErrorInvalidConfiguration;
    }
    cudaLaunchConfig_t q = {};
    q.gridDim = dim3(2);
    q.blockDim = dim3(num_threads<kEpi>());
    q.dynamicSmemBytes = smem;
    cudaLaunchAttribute ca[1];
    ca[0].id = cudaLaunchAttributeClusterDimension;
    ca[0].val.clusterDim.x = 2;
    ca[0].val.clusterDim.y = 1;
    ca[0].val.clusterDim.z = 1;
    q.attrs = ca;
    q.numAttrs = 1;
    int n = 0;
    e = cudaOccupancyMaxActiveClusters(&n, kernel, &q);
    if (e != cudaSuccess) return e;
    if (n < 1) return cudaErrorInvalidConfiguration;
    max_pairs = n;
  }
  const int tiles = ((p.M + 255) / 256) * ((p.N + BN - 1) / BN);
  const int pairs = tiles < max_pairs ? tiles : max_pairs;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs);
  cfg.blockDim = dim3(num_threads<kEpi>());
  cfg.dynamicSmemBytes = smem;
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
  return cudaLaunchKernelEx(&cfg, kernel, t.a, t.b, t.la, t.lb, t.y, t.sfa, t.sfb, tm_x, tm_l1, p);
}
}  // namespace

cudaError_t launch_gemm_nvfp4_pair(const GemmNvfp4Params& p, const GemmPairTmaps& t, cudaStream_t stream, bool pdl) {
  return launch_pair_impl<EPI_PLAIN, false>(p, t, t.a, t.a, stream, pdl);
}

cudaError_t launch_gemm_nvfp4_pair_gelu(const GemmNvfp4Params& p, const GemmPairTmaps& t, cudaStream_t stream,
                                        bool pdl) {
  return launch_pair_impl<EPI_GELU, false>(p, t, t.a, t.a, stream, pdl);
}

cudaError_t launch_gemm_nvfp4_pair_qkv(const GemmNvfp4Params& p, const GemmPairTmaps& t, cudaStream_t stream,
                                       bool pdl) {
  return launch_pair_impl<EPI_QKV, false>(p, t, t.a, t.a, stream, pdl);
}

cudaError_t launch_gemm_f16_pair(const GemmNvfp4Params& p, const GemmPairTmaps& t, cudaStream_t stream, bool pdl) {
  return launch_pair_impl<EPI_F16, false>(p, t, t.a, t.a, stream, pdl);
}

cudaError_t launch_layer_nvfp4_pair(const GemmNvfp4Params& p, const GemmPairTmaps& t, const CUtensorMap& tm_x,
                                    const CUtensorMap& tm_l1, cudaStream_t stream, bool pdl) {
  return launch_pair_impl<EPI_PLAIN, true>(p, t, tm_x, tm_l1, stream, pdl);
}

}  // namespace svdq
