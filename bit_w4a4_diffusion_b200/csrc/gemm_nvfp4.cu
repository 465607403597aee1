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

#include "epilogue.cuh"
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
constexpr int EPI_CHUNK = 16;                          // columns per TMEM load / store
constexpr int EPI_BUF_BYTES = 32 * EPI_CHUNK * 2;      // 32 rows x 32 B
constexpr int EPI_BYTES = 4 * 2 * EPI_BUF_BYTES;       // epilogue staging, 8 KB

// Warp roles.  Plain epilogue (9 warps): producer 0, MMA 1, epilogue 2-5,
// block-scale copies 6-8.  GELU-MLP epilogue (12 warps, three warpgroups):
// epilogue 0-7, producer 8, MMA 9, block-scale copies 10-11; the last
// warpgroup hands registers to the two epilogue warpgroups (setmaxnreg).
// Epilogue kinds: y = bf16(alpha D + b); the GELU-MLP epilogue; the QKV
// epilogue with RMSNorm and RoPE.  The last two use the wide layout.
constexpr int EPI_PLAIN = 0, EPI_GELU = 1, EPI_QKV = 2;
template <bool kWide>
struct Roles {
  static constexpr int EPI_WARPS = kWide ? 8 : 4;
  static constexpr int PRODUCER = kWide ? 8 : 0;
  static constexpr int MMA = kWide ? 9 : 1;
  static constexpr int SF_W0 = kWide ? 10 : 6;
  static constexpr int SF_WARPS = kWide ? 2 : 3;
  static constexpr int NUM_THREADS = (kWide ? 12 : 9) * 32;
};
// Register split of the wide layout: launched at 168 per thread
// (12 warps x 32 x 168 = 64512), then 216 for each epilogue thread and 72 for
// the rest: 256 x 216 + 128 x 72 = 64512.
constexpr int GQ_LAUNCH_REGS = 168, GQ_EPI_REGS = 216, GQ_CTL_REGS = 72;
static_assert(256 * GQ_EPI_REGS + 128 * GQ_CTL_REGS <= 384 * GQ_LAUNCH_REGS, "register split");
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

// The GELU-MLP epilogue keeps the tile's 1/lambda (fp32) and bias (bf16)
// columns in shared memory after the staging buffers.
constexpr int GQ_TABLE_BYTES = BN * 4 + BN * 2;
template <int kEpi>
constexpr size_t smem_bytes() {
  return 1024 /*align slack*/ + STAGES * STAGE_BYTES + EPI_BYTES + (kEpi != EPI_PLAIN ? GQ_TABLE_BYTES : 0) +
         sizeof(SmemCtl);
}
static_assert(smem_bytes<EPI_GELU>() <= 232448, "shared memory per block");

// Instruction descriptors (tcgen05 "instruction descriptor" bit fields).
//   block-scaled: a/b format E2M1 (=1) at bits 7/10, N>>3 at 17, UE4M3 scales
//   (bit 23 = 0), M>>4 at 24.  f16 kind: f32 accumulate (bit 4), bf16 a/b (=1).
constexpr uint32_t IDESC_NVFP4 = (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
constexpr uint32_t IDESC_BF16 =
    (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);

SVDQ_DEV uint64_t sw128_desc(uint32_t saddr) { return smem_desc(saddr, 16, 1024, 2); }
SVDQ_DEV uint64_t sf_desc(uint32_t saddr) { return smem_desc(saddr, 0, 128, 0); }

template <int kEpi>
__global__ void __launch_bounds__(Roles<kEpi != EPI_PLAIN>::NUM_THREADS, 1)
    gemm_nvfp4_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                      const __grid_constant__ CUtensorMap tm_la, const __grid_constant__ CUtensorMap tm_lb,
                      const __grid_constant__ CUtensorMap tm_y, const GemmNvfp4Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stage_base = smem;
  uint8_t* epi_base = smem + STAGES * STAGE_BYTES;
  constexpr bool kGelu = kEpi == EPI_GELU, kQkv = kEpi == EPI_QKV, kWide = kEpi != EPI_PLAIN;
  SmemCtl* ctl = reinterpret_cast<SmemCtl*>(epi_base + EPI_BYTES + (kWide ? GQ_TABLE_BYTES : 0));

  using R = Roles<kWide>;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles_m = (p.M + BM - 1) / BM;
  const int tiles_n = (p.N + BN - 1) / BN;
  const int num_tiles = tiles_m * tiles_n;
  const int k_tiles = p.K / 256;
  const int slices = k_tiles + 1;  // + the low-rank slice
  // Tile schedule.  Plain epilogue: round robin over tiles numbered M-block
  // fastest.  GELU-MLP epilogue: CTA i takes the contiguous run
  // [i T / G, (i + 1) T / G) of tiles numbered N-block fastest, so that its
  // consecutive tiles share an M-block and the epilogue can carry the
  // low-rank partial of those rows from tile to tile.  (All operands of one
  // layer fit in L2, so the order does not change DRAM traffic.)
  const int t_begin = kGelu ? (int)((long long)blockIdx.x * num_tiles / gridDim.x) : (int)blockIdx.x;
  const int t_end = kGelu ? (int)((long long)(blockIdx.x + 1) * num_tiles / gridDim.x) : num_tiles;
  const int t_step = kGelu ? 1 : (int)gridDim.x;
  auto tile_m0 = [&](int tile) { return (kGelu ? tile / tiles_n : tile % tiles_m) * BM; };
  auto tile_n0 = [&](int tile) { return (kGelu ? tile % tiles_n : tile / tiles_m) * BN; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&ctl->full[s]), 1);
      mbar_init(smem_u32(&ctl->empty[s]), 1);
    }
    mbar_init(smem_u32(&ctl->acc_full), 1);
    mbar_init(smem_u32(&ctl->acc_empty), R::EPI_WARPS);
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&ctl->sf_full[b]), R::SF_WARPS);
      mbar_init(smem_u32(&ctl->sf_empty[b]), 1);
    }
    mbar_init(smem_u32(&ctl->drain), 1);
    mbar_init(smem_u32(&ctl->sf_drain), R::SF_WARPS);
    ctl->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == R::PRODUCER && lane == 0) {
    prefetch_tmap(&tm_a);
    prefetch_tmap(&tm_b);
    prefetch_tmap(&tm_la);
    prefetch_tmap(&tm_lb);
    if (kEpi == EPI_PLAIN) prefetch_tmap(&tm_y);
  }
  if (warp == R::MMA) {
    tmem_alloc(smem_u32(&ctl->tmem_base), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;

  // Inputs produced by the preceding quantize kernel become visible here.
  pdl_wait();
  // The next kernel on the stream may be scheduled from now on; it waits for
  // this grid's completion before it reads anything.
  pdl_launch_dependents();

  WaitCtx wctx{&ctl->abort_flag, p.dev_status, p.timeout_ns};

  // ---------------------------------------------------------------- roles
  // Role loops run on the whole warp and issue from one elected lane (the
  // lowest, the same one every time): tcgen05 and TMA instructions take
  // uniform-register operands, which a loop run by lane 0 alone does not
  // keep, and each issue then costs several times more.
  auto role_producer = [&]() {
    {
      // ------------------------------------------------------------ producer
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_phase = 0;  // per stage: load outstanding, its parity
      bool ok = true;
      const uint64_t pol_w = policy_evict_last();
      for (int tile = t_begin; tile < t_end && ok; tile += t_step) {
        const int m0 = tile_m0(tile);
        const int n0 = tile_n0(tile);
        for (int kt = 0; kt < slices; ++kt) {
          if (!mbar_wait_warp(smem_u32(&ctl->empty[stage]), phase ^ 1, wctx, kDevTimeoutProducer)) {
            ok = false;
            break;
          }
          uint8_t* sa = stage_base + stage * STAGE_BYTES;
          uint8_t* sb = sa + A_BYTES;
          uint8_t* ssfa = sb + B_BYTES;
          uint8_t* ssfb = ssfa + SFA_BYTES;
          const uint32_t full = smem_u32(&ctl->full[stage]);
          if (!elect_one()) {
          } else if (kt == 0) {
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
          __syncwarp();
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
  };
  auto role_mma = [&]() {
    {
      // ------------------------------------------------------------ MMA issuer
      int stage = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      int it = 0;
      uint32_t ks = 0;  // K slices computed so far (selects the scale buffer)
      for (int tile = t_begin; tile < t_end && ok; tile += t_step, ++it) {
        const uint32_t d_tmem = tmem + (uint32_t)((it & 1) * ACC_STRIDE);
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
          if (kt == 0) {
            if (elect_one()) {
#pragma unroll
              for (int j = 0; j < 4; ++j)
                mma_bf16(d_tmem, sw128_desc(sa + 32 * j), sw128_desc(sb + 32 * j), IDESC_BF16, j > 0 ? 1u : 0u);
            }
            __syncwarp();
          } else {
            const uint32_t buf = ks & 1;
            if (!mbar_wait_warp(smem_u32(&ctl->sf_full[buf]), (ks >> 1) & 1, wctx, kDevTimeoutMma)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t sf = tmem + TMEM_SF0 + buf * SF_COLS;
            if (elect_one()) {
#pragma unroll
              for (int j = 0; j < 4; ++j)
                mma_nvfp4(d_tmem, sw128_desc(sa + 32 * j), sw128_desc(sb + 32 * j), IDESC_NVFP4,
                          sf + TMEM_SFA_OFF + 4 * j, sf + TMEM_SFB_OFF + 8 * j, 1u);
              tc_commit(smem_u32(&ctl->sf_empty[buf]));
            }
            __syncwarp();
            ++ks;
          }
          if (elect_one()) tc_commit(smem_u32(&ctl->empty[stage]));
          __syncwarp();
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        if (elect_one()) tc_commit(smem_u32(&ctl->acc_full));
        __syncwarp();
        acc_phase ^= 1;
      }
      // Wait for every MMA the elected lane issued before TMEM is freed.
      if (elect_one()) tc_commit(smem_u32(&ctl->drain));
      __syncwarp();
      volatile int never = 0;
      WaitCtx drain_ctx{&never, p.dev_status, kDrainLimitNs};
      mbar_wait(smem_u32(&ctl->drain), 0, drain_ctx, kDevTimeoutDrain);
    }
  };
  auto role_scale_copies = [&]() {
    {
      // ------------------------------------------------------------ scale copies
      // Three jobs per K slice: 0 = SFA (4 copies), 1 / 2 = SFB rows 0-127 /
      // 128-255 (4 each); scale-copy warp w takes jobs w, w + SF_WARPS, ...
      const int w = warp - R::SF_W0;
      int stage = 0;
      uint32_t phase = 0, ks = 0;
      bool ok = true;
      for (int tile = t_begin; tile < t_end && ok; tile += t_step) {
        for (int kt = 0; kt < slices; ++kt) {
          if (kt > 0) {
            const uint32_t buf = ks & 1;
            // The MMAs of the K slice two back read this buffer; wait for them.
            if (ks >= 2 &&
                !mbar_wait_warp(smem_u32(&ctl->sf_empty[buf]), ((ks - 2) >> 1) & 1, wctx, kDevTimeoutMma)) {
              ok = false;
              break;
            }
            if (!mbar_wait_warp(smem_u32(&ctl->full[stage]), phase, wctx, kDevTimeoutMma)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t ssfa = smem_u32(stage_base + stage * STAGE_BYTES) + A_BYTES + B_BYTES;
            const bool leader = elect_one();
            for (int job = w; job < 3 && leader; job += R::SF_WARPS) {
              const uint32_t src = job == 0 ? ssfa : ssfa + SFA_BYTES * job;
              const uint32_t dst =
                  tmem + TMEM_SF0 + buf * SF_COLS + (job == 0 ? TMEM_SFA_OFF : TMEM_SFB_OFF + 4 * (job - 1));
              const uint32_t col_step = job == 0 ? 4 : 8;
#pragma unroll
              for (int j = 0; j < 4; ++j) tmem_cp_32x128_warpx4(dst + col_step * j, sf_desc(src + 512 * j));
            }
            if (leader) tc_commit(smem_u32(&ctl->sf_full[buf]));
            __syncwarp();
            ++ks;
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (elect_one()) tc_commit(smem_u32(&ctl->sf_drain));
      __syncwarp();
      volatile int never = 0;
      WaitCtx drain_ctx{&never, p.dev_status, kDrainLimitNs};
      mbar_wait(smem_u32(&ctl->sf_drain), 0, drain_ctx, kDevTimeoutDrain);
    }
  };
  auto role_epilogue = [&]() {
    if constexpr (kGelu) {
    // ------------------------------------------------------ GELU-MLP epilogue
    // Eight warps: warp w reads TMEM lane quarter w mod 4 (32 rows) and one
    // half of the tile's eight 32-column chunks (w / 4 = 0: the first four in
    // the ring order below, which include the columns shared with the other
    // accumulator; 1: the last four), each by gelu_quant_chunk (epilogue.cuh:
    // GELU, the down layer's quantizer, its low-rank partials).  The tile's
    // 1/lambda and bias columns are staged once per tile in shared memory.
    // The partial sums of consecutive tiles of one M-block stay in registers
    // and go to u_work with vector reductions when the M-block changes (fire
    // and forget: the conversion to lora_act is a separate kernel that runs
    // after this grid).  The eight warps share named barriers 2 and 3,
    // so every stop decision is taken by all of them.
    constexpr int NT = R::EPI_WARPS * 32;
    const int q = warp & 3, hf = warp >> 2;
    const int g = lane >> 2, c = lane & 3;
    const int et = threadIdx.x;  // 0..255 over the epilogue warps
    const GeluQuantParams& gq = p.gq;
    const uint32_t hbase = smem_u32(epi_base + warp * 1024);
    float* tab_inv = reinterpret_cast<float*>(epi_base + EPI_BYTES);
    uint16_t* tab_bias = reinterpret_cast<uint16_t*>(epi_base + EPI_BYTES + BN * 4);
    const float2 lr2 = make_float2(gq.lr_in_scale, gq.lr_in_scale);
    const float2 alpha2 = make_float2(p.alpha, p.alpha);
    const float inv_six_s = __frcp_rn(__fmul_rn(6.0f, gq.s_d));
    const GeluLane L{tab_inv, tab_bias, alpha2, lr2, inv_six_s, hbase, lane, g, c};
    uint32_t acc_phase = 0;
    int it = 0;
    constexpr int LDC = 32;
    constexpr int NCH = BN / LDC;
    constexpr int NSH = (ACC_OVERLAP + LDC - 1) / LDC;
    constexpr int CPW = NCH / 2;  // chunks per warp
    constexpr int NBUF = 3;
    static_assert(NSH <= NBUF && NBUF <= CPW, "the shared chunks fit the first ring fill of half 0");
    // The warp's low-rank partial of its 32 rows: rows 16t + g (+8), ranks
    // 8j + 2c (+1); added into u_work when the M-block changes and at the end.
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
    for (int tile = t_begin; tile < t_end; tile += t_step, ++it) {
      const int m0 = tile_m0(tile);
      const int n0 = tile_n0(tile);
      const int b = it & 1;
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
      const uint32_t acc_base = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(b * ACC_STRIDE);
      // Ring order: the shared columns first (the last ACC_OVERLAP of
      // accumulator 0, the first ACC_OVERLAP of accumulator 1).
      auto chunk_col = [&](int i) { return b == 0 ? (i + NCH - NSH) % NCH : i; };
      const int i0 = hf * CPW;
      uint32_t rb[NBUF][32];
#pragma unroll
      for (int i = 0; i < NBUF; ++i) tmem_ld_32x32b_x32(acc_base + chunk_col(i0 + i) * LDC, rb[i]);
      tmem_ld_wait(rb[0]);
      reg_fence(rb[1]);
      reg_fence(rb[2]);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&ctl->acc_empty));
#pragma unroll
      for (int ii = 0; ii < CPW; ++ii) {
        uint32_t(&r)[32] = rb[ii % NBUF];
        if (ii >= NBUF && ii % NBUF == 0) {
          tmem_ld_wait(rb[0]);
          reg_fence(rb[1]);
          reg_fence(rb[2]);
        }
        const int cl = chunk_col(i0 + ii) * LDC;  // column within the tile
        gelu_quant_chunk(r, L, gq, p.N, cl, n0 + cl, row, row_ok, lacc);
        // Refill the block just converted with the chunk three ahead.
        if (ii + NBUF < CPW) tmem_ld_32x32b_x32(acc_base + chunk_col(i0 + ii + NBUF) * LDC, r);
      }
      acc_phase ^= 1;
    }
    if (cur_m0 >= 0) flush_lacc(cur_m0);
    } else if constexpr (kQkv) {
      // ------------------------------------------ QKV + RMSNorm + RoPE epilogue
      // Eight warps: warp w reads TMEM lane quarter w mod 4 (32 rows) and head
      // w / 4 of the tile (a 256-column tile holds two 128-feature heads).  A
      // lane loads its row's whole head (128 registers) before the warp
      // releases the accumulator, so the head holding the columns shared with
      // the other accumulator is read in full first; qkv_head (epilogue.cuh)
      // does the rest.  The gamma vectors (for the whole kernel) and the
      // tile's bias columns sit in shared memory; the rotary tables are
      // pair-major ([64][M]), so that the 32 rows of a warp read one line per
      // pair.
      constexpr int NT = R::EPI_WARPS * 32;
      const int q = warp & 3, hf = warp >> 2;
      const int et = threadIdx.x;  // 0..255 over the epilogue warps
      const QkvParams& qp = p.qk;
      const float2 alpha2 = make_float2(p.alpha, p.alpha);
      float* tab_g = reinterpret_cast<float*>(epi_base + EPI_BYTES);                  // gamma_q | gamma_k
      uint16_t* tab_bias = reinterpret_cast<uint16_t*>(epi_base + EPI_BYTES + 1024);  // 256 bf16
      const uint32_t slab = smem_u32(epi_base + warp * 1024);
      tab_g[et] = et < 128 ? __ldg(qp.gamma_q + et) : __ldg(qp.gamma_k + et - 128);
      uint32_t acc_phase = 0;
      int it = 0;
      for (int tile = t_begin; tile < t_end; tile += t_step, ++it) {
        const int m0 = tile_m0(tile);
        const int n0 = tile_n0(tile);
        const int b = it & 1;
        const int row = m0 + 32 * q + lane;
        const bool row_ok = row < p.M;
        const int n = n0 + 128 * hf;  // first column of this warp's head
        const bool head_ok = n < p.N;
        const uint16_t my_bias = (p.bias != nullptr && n0 + et < p.N) ? __ldg(p.bias + n0 + et) : (uint16_t)0;
        const bool got = mbar_wait(smem_u32(&ctl->acc_full), acc_phase, wctx, kDevTimeoutEpilogue);
        // All epilogue threads decide together; this barrier also ends every
        // read of the previous tile's bias columns.
        if (named_bar_any(2, NT, !got)) break;
        tab_bias[et] = my_bias;
        asm volatile("bar.sync 3, %0;" ::"n"(NT) : "memory");
        tc_fence_after();
        const uint32_t acc_base = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(b * ACC_STRIDE + 128 * hf);
        uint32_t r[4][32];
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) tmem_ld_32x32b_x32(acc_base + 32 * c4, r[c4]);
        tmem_ld_wait(r[0]);
        reg_fence(r[1]);
        reg_fence(r[2]);
        reg_fence(r[3]);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&ctl->acc_empty));
        acc_phase ^= 1;
        if (!head_ok) continue;
        const int part = n / qp.hd;  // 0: Q, 1: K, 2: V
        qkv_head(r, tab_bias + 128 * hf, tab_g + 128 * (part < 2 ? part : 0), alpha2, qp, part, p.M, p.N, row,
                 row_ok, m0 + 32 * q, n, slab, lane);
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
    uint8_t* buf0 = epi_base + (warp - 2) * 2 * EPI_BUF_BYTES;  // epilogue warps 2-5
    uint32_t acc_phase = 0;
    int chunk_seq = 0, it = 0;
    constexpr int LDC = 32;                    // columns per TMEM load
    constexpr int NCH = BN / LDC;
    constexpr int NSH = (ACC_OVERLAP + LDC - 1) / LDC;  // chunks holding shared columns
    constexpr int NBUF = 3;
    static_assert(NSH <= NBUF, "the shared chunks fit the first ring fill");
    for (int tile = t_begin; tile < t_end; tile += t_step, ++it) {
      const int m0 = tile_m0(tile);
      const int n0 = tile_n0(tile);
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
  };

  if constexpr (kWide) {
    // setmaxnreg is warpgroup-wide: the last warpgroup (producer, MMA, scale
    // copies) gives registers to the two epilogue warpgroups.
    if (warp >= R::EPI_WARPS) {
      asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(GQ_CTL_REGS));
      if (warp == R::PRODUCER)
        role_producer();
      else if (warp == R::MMA)
        role_mma();
      else
        role_scale_copies();
    } else {
      asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(GQ_EPI_REGS));
      role_epilogue();
    }
  } else {
    if (warp == R::PRODUCER)
      role_producer();
    else if (warp == R::MMA)
      role_mma();
    else if (warp >= R::SF_W0)
      role_scale_copies();
    else
      role_epilogue();
  }


  tc_fence_before();
  __syncthreads();
  if (warp == R::MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace

namespace {
template <int kEpi>
cudaError_t launch_impl(const GemmNvfp4Params& p, const GemmTmaps& t, int num_sms, cudaStream_t stream, bool pdl) {
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(gemm_nvfp4_kernel<kEpi>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem_bytes<kEpi>());
    if (e != cudaSuccess) return e;
    if (kEpi != EPI_PLAIN) {
      // The epilogue warpgroups' setmaxnreg.inc waits until the others have
      // released enough registers: only launch if the compiled register
      // count makes the split add up.
      cudaFuncAttributes fa;
      e = cudaFuncGetAttributes(&fa, gemm_nvfp4_kernel<kEpi>);
      if (e != cudaSuccess) return e;
      if (fa.numRegs * Roles<true>::NUM_THREADS < 256 * GQ_EPI_REGS + 128 * GQ_CTL_REGS)
        return cudaErrorInvalidConfiguration;
    }
    attr_set = true;
  }
  const int tiles = ((p.M + BM - 1) / BM) * ((p.N + BN - 1) / BN);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(tiles < num_sms ? tiles : num_sms);
  cfg.blockDim = dim3(Roles<kEpi != EPI_PLAIN>::NUM_THREADS);
  cfg.dynamicSmemBytes = smem_bytes<kEpi>();
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, gemm_nvfp4_kernel<kEpi>, t.a, t.b, t.la, t.lb, t.y, p);
}
}  // namespace

cudaError_t launch_gemm_nvfp4(const GemmNvfp4Params& p, const GemmTmaps& t, int num_sms, cudaStream_t stream,
                              bool pdl) {
  return launch_impl<EPI_PLAIN>(p, t, num_sms, stream, pdl);
}

cudaError_t launch_gemm_nvfp4_gelu(const GemmNvfp4Params& p, const GemmTmaps& t, int num_sms, cudaStream_t stream,
                                   bool pdl) {
  return launch_impl<EPI_GELU>(p, t, num_sms, stream, pdl);
}

cudaError_t launch_gemm_nvfp4_qkv(const GemmNvfp4Params& p, const GemmTmaps& t, int num_sms, cudaStream_t stream,
                                  bool pdl) {
  return launch_impl<EPI_QKV>(p, t, num_sms, stream, pdl);
}

namespace {
// lora_act[m] = [hi(u c) | lo(u c)] with u the summed low-rank partials.
__global__ void __launch_bounds__(256) lowrank_finalize_kernel(const float* __restrict__ u_work, int M, float c,
                                                              uint16_t* __restrict__ lora_act) {
  pdl_wait();
  pdl_launch_dependents();
  const int i = blockIdx.x * 256 + threadIdx.x;
  if (i >= M * 32) return;
  const int m = i >> 5, col = i & 31;
  const float uf = __fmul_rn(u_work[i], c);
  const __nv_bfloat16 hi = __float2bfloat16_rn(uf);
  const __nv_bfloat16 lo = __float2bfloat16_rn(__fsub_rn(uf, __bfloat162float(hi)));
  lora_act[(size_t)m * 64 + col] = __bfloat16_as_ushort(hi);
  lora_act[(size_t)m * 64 + 32 + col] = __bfloat16_as_ushort(lo);
}
}  // namespace

cudaError_t launch_lowrank_finalize(const float* u_work, int M, float lora_scale, uint16_t* lora_act,
                                    cudaStream_t stream, bool pdl) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((M * 32 + 255) / 256));
  cfg.blockDim = dim3(256);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, lowrank_finalize_kernel, u_work, M, lora_scale, lora_act);
}

}  // namespace svdq
