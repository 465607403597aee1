// S3 of the INT4 layer on CTA pairs, with the 4-bit operands dequantized to
// fp16 inside the GEMM: the product on the fp16 tensor pipe without an fp16
// copy of either operand in memory (opt-in, SVDQ_INT4_LAYER_GEMM=dq).  It
// gives the same y as the default path (both operands written out in fp16
// first, then gemm_nvfp4_pair.cu's fp16 path) bit for bit, and is slower on
// B200: 229 against 105 us at M = 4096, K = N = 3072.  Two costs, measured
// with timing-only copies: CTA 1's release arrive on CTA 0's barrier after
// every K slice stalls its dequantization warps (about 78 us of the 229; a
// relaxed arrive, which orders nothing, gave 151 us), and four warps
// converting 16 KB of codes into 32 KB of swizzled fp16 per K slice do not
// keep up with the MMAs (the 151 us).
//
// Pages: "Nunchaku Lite" docs, "Supported quantization types" table
// (svdq_w4a4, int4, group 64) and its tip that int4 checkpoints on Blackwell
// may be slower than nvfp4: these tensor cores have no 4-bit integer MMA.
// "Hugging Face integrates Nunchaku 4-bit diffusion inference into
// Diffusers", section "SVDQuant and the Nunchaku engine": the low-rank
// up-projection is fused into the 4-bit GEMM.
//
//   D[m,n] = sum_k A'[m,k] W'[n,k] + la'[m,:] . lb'[n,:]            (fp32, TMEM)
//   A'[m,k] = fp16(sa[m,k/64] 2^-Ea[m] qa[m,k]),  W' likewise with Ew[n]
//   la' = lora_act 2^-Ea[m],  lb' = [L2^T|L2^T] 2^-Ew[n]             (bf16, exact)
//   y[m,n]  = bf16(D[m,n] 2^Ea[m] 2^Ew[n] + bias[n])
//
// The exactness argument and the row exponents E are those of
// dequant_int4.cu, which computes 2^E and the scaled low-rank rows in a small
// pass over the scales before this kernel (its factor-only mode).  Here each
// K slice is one 64-group: the producer copies the slice's packed codes (32
// bytes per row) and the group's bf16 scale of each row into shared memory,
// and four dequantization warps turn them into the SWIZZLE_128B K-major fp16
// operand tiles the MMA reads (thread t: row t of A and row t of this CTA's
// half of B; 64 codes -> 128 bytes each, same (0,2,4,6,1,3,5,7) order within
// every 8 codes for both operands, so the dot products are unchanged).
//
// A cluster of two CTAs computes a 256 x 256 output tile (tcgen05
// .cta_group::2, M = 256): CTA r holds rows [128 r, +128) of the A tile and
// rows [128 r, +128) of the B tile, as in gemm_nvfp4_pair.cu.  Tensor memory
// holds one accumulator (256 columns).
//
// Roles (16 warps per CTA; the four warpgroups split the registers with
// setmaxnreg: the epilogue warpgroups rise to 168, the others drop to 88):
//   warps 0..7    epilogue, both CTAs: warp w reads TMEM lane quarter w % 4,
//                 columns [128 (w / 4), +128)
//   warp 8        producer, both CTAs: codes by TMA, scales by bulk copy,
//                 into its own CTA's stage; the low-rank slice's scaled
//                 operands by TMA straight into the operand tiles
//   warp 9        CTA 0: MMAs for the pair
//   warps 10, 11  idle
//   warps 12..15  dequantization, both CTAs
// Synchronisation:
//   raw_full[s]   each CTA, local: the stage's copies landed
//   opnd_full[s]  CTA 0, two arrivals: each CTA's dequantization warps
//                 announce their operand tiles (release at cluster scope
//                 after a proxy fence, so the tensor core sees the writes)
//   empty[s]      both CTAs: the MMA warp's commit multicasts to both
//   acc_full      both CTAs; acc_empty CTA 0 (16 epilogue warps arrive)
// Every wait is bounded; on timeout the kernel records a status code, stops
// every role, drains its own copies and MMAs, and both CTAs meet at the
// final cluster barrier.
#include <cuda_bf16.h>
#include <cstdint>

#include "int4_fp16.cuh"
#include "ptx.cuh"
#include "svdq_internal.h"

namespace svdq {
namespace {

constexpr int BM = 128;                           // rows per CTA
constexpr int BN = 256;                           // output columns per tile
constexpr int BN_HALF = BN / 2;                   // B rows per CTA
constexpr int KS = 64;                            // K elements per slice: one 64-group
constexpr int STAGES = 5;
constexpr int A16_BYTES = BM * KS * 2;            // 16 KB fp16 operand tile
constexpr int B16_BYTES = BN_HALF * KS * 2;       // 16 KB
constexpr int A4_BYTES = BM * KS / 2;             // 4 KB packed codes
constexpr int B4_BYTES = BN_HALF * KS / 2;        // 4 KB
constexpr int SC_BYTES = 1024;                    // bf16 scales: A [128] at 0, B [128] at 256
constexpr int STAGE_BYTES = A16_BYTES + B16_BYTES + A4_BYTES + B4_BYTES + SC_BYTES;
static_assert(STAGE_BYTES % 1024 == 0, "stages keep the 1024-byte alignment of SWIZZLE_128B");
constexpr int RAW_BYTES = A4_BYTES + B4_BYTES + 2 * 256;   // one K slice's copies per CTA
constexpr int EPI_WARPS = 8;
constexpr int PRODUCER_WARP = 8;
constexpr int MMA_WARP = 9;
constexpr int DQ_WARP0 = 12;
constexpr int DQ_THREADS = 128;
constexpr int NUM_THREADS = 16 * 32;
constexpr int LAUNCH_REGS = 128, EPI_REGS = 168, CTL_REGS = 88;
static_assert(256 * EPI_REGS + 256 * CTL_REGS <= NUM_THREADS * LAUNCH_REGS, "register split");
constexpr int EPI_COLS = BN / 2;                  // columns per epilogue warp
constexpr int EPI_CHUNK = 16;                     // columns per TMA store
constexpr int EPI_BUF_BYTES = 32 * EPI_CHUNK * 2;
constexpr int EPI_BYTES = EPI_WARPS * 2 * EPI_BUF_BYTES;
constexpr int TMEM_COLS = 256;
constexpr uint16_t PAIR_MASK = 0x3;
constexpr unsigned long long kDrainLimitNs = 2000000000ull;

struct SmemCtl {
  uint64_t raw_full[STAGES];
  uint64_t opnd_full[STAGES];
  uint64_t empty[STAGES];
  uint64_t acc_full;
  uint64_t acc_empty;
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

constexpr size_t SMEM_BYTES = 1024 + (size_t)STAGES * STAGE_BYTES + EPI_BYTES + sizeof(SmemCtl);
static_assert(SMEM_BYTES <= 232448, "fits the 227 KB opt-in shared memory of one CTA");

// Instruction descriptors for M = 256 (the pair), N = 256, fp32 D: fp16
// operands for the K slices, bf16 for the low-rank slice.
constexpr uint32_t IDESC_F16 = (1u << 4) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(256 >> 4) << 24);
constexpr uint32_t IDESC_BF16 = IDESC_F16 | (1u << 7) | (1u << 10);

SVDQ_DEV uint64_t sw128_desc(uint32_t saddr) { return smem_desc(saddr, 16, 1024, 2); }

SVDQ_DEV float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
SVDQ_DEV float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

SVDQ_DEV uint4 lds_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}
SVDQ_DEV void sts_v4(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}
SVDQ_DEV uint32_t lds_u16(uint32_t addr) {
  unsigned short v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr));
  return v;
}
// Arrive on an mbarrier given by its shared::cluster address, with release
// semantics at cluster scope: the arriving thread's earlier writes (and,
// through the preceding CTA barrier, those of the threads it synchronised
// with) are visible to a thread that observes the phase with acquire.
SVDQ_DEV void mbar_arrive_cluster_release(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// One operand row: 64 codes (32 bytes at `codes`) times the row's scaled
// group scale -> 128 bytes in row r of a SWIZZLE_128B K-major tile at `tile`
// (16-byte chunk c of row r at r * 128 + ((c ^ (r mod 8)) * 16)).
SVDQ_DEV void dequant_row(uint32_t codes, uint32_t s2, uint32_t tile, int r) {
  const uint4 w0 = lds_v4(codes), w1 = lds_v4(codes + 16);
  const uint32_t w[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
  const uint32_t row = tile + (uint32_t)r * 128u;
#pragma unroll
  for (int c = 0; c < 8; ++c) sts_v4(row + (uint32_t)((c ^ (r & 7)) << 4), i4_dequant_word(w[c], s2));
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
    gemm_int4_pair_kernel(const __grid_constant__ CUtensorMap tm_a4, const __grid_constant__ CUtensorMap tm_b4,
                          const __grid_constant__ CUtensorMap tm_la, const __grid_constant__ CUtensorMap tm_lb,
                          const __grid_constant__ CUtensorMap tm_y, const GemmInt4DqParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* epi_base = smem + STAGES * STAGE_BYTES;
  SmemCtl* ctl = reinterpret_cast<SmemCtl*>(epi_base + EPI_BYTES);
  auto a16 = [&](int s) { return smem + s * STAGE_BYTES; };
  auto b16 = [&](int s) { return smem + s * STAGE_BYTES + A16_BYTES; };
  auto a4 = [&](int s) { return smem + s * STAGE_BYTES + A16_BYTES + B16_BYTES; };
  auto b4 = [&](int s) { return smem + s * STAGE_BYTES + A16_BYTES + B16_BYTES + A4_BYTES; };
  auto scl = [&](int s) { return smem + s * STAGE_BYTES + A16_BYTES + B16_BYTES + A4_BYTES + B4_BYTES; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();     // 0: leader (issues the MMAs), 1: peer
  const int pair = blockIdx.x >> 1, num_pairs = gridDim.x >> 1;
  const int tiles_m = (p.M + 2 * BM - 1) / (2 * BM);
  const int tiles_n = (p.N + BN - 1) / BN;
  const int num_tiles = tiles_m * tiles_n;
  const int slices = p.K / KS + 1;             // + the low-rank slice (slice 0)
  auto tile_m0 = [&](int tile) { return (tile % tiles_m) * 2 * BM + (int)rank * BM; };
  auto tile_n0 = [&](int tile) { return (tile / tiles_m) * BN; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&ctl->raw_full[s]), 1);
      mbar_init(smem_u32(&ctl->opnd_full[s]), 2);
      mbar_init(smem_u32(&ctl->empty[s]), 1);
    }
    mbar_init(smem_u32(&ctl->acc_full), 1);
    mbar_init(smem_u32(&ctl->acc_empty), 2 * EPI_WARPS);
    mbar_init(smem_u32(&ctl->drain), 1);
    ctl->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == PRODUCER_WARP && lane == 0) {
    prefetch_tmap(&tm_a4);
    prefetch_tmap(&tm_b4);
    prefetch_tmap(&tm_la);
    prefetch_tmap(&tm_lb);
    prefetch_tmap(&tm_y);
  }
  if (warp == MMA_WARP) {
    tmem_alloc_pair(smem_u32(&ctl->tmem_base), TMEM_COLS);
    tmem_relinquish_pair();
  }
  __syncwarp();
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;

  pdl_wait();
  pdl_launch_dependents();

  WaitCtx wctx{&ctl->abort_flag, p.dev_status, p.timeout_ns};

  if (warp >= EPI_WARPS) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(CTL_REGS));
    if (warp == PRODUCER_WARP) {
      // ------------------------------------------------------------ producer
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_phase = 0;
      bool ok = true;
      const uint64_t pol = policy_evict_last();   // every operand is re-read by other tiles
      for (int tile = pair; tile < num_tiles && ok; tile += num_pairs) {
        const int m0 = tile_m0(tile);
        const int nb = tile_n0(tile) + (int)rank * BN_HALF;
        for (int kt = 0; kt < slices; ++kt) {
          if (!mbar_wait_warp(smem_u32(&ctl->empty[stage]), phase ^ 1, wctx, kDevTimeoutProducer)) {
            ok = false;
            break;
          }
          if (elect_one()) {
            const uint32_t full = smem_u32(&ctl->raw_full[stage]);
            if (kt == 0) {
              mbar_arrive_expect_tx(full, A16_BYTES + B16_BYTES);
              tma_load_2d_hint(smem_u32(a16(stage)), &tm_la, 0, m0, full, pol);
              tma_load_2d_hint(smem_u32(b16(stage)), &tm_lb, 0, nb, full, pol);
            } else {
              const int g = kt - 1;
              mbar_arrive_expect_tx(full, RAW_BYTES);
              tma_load_2d_hint(smem_u32(a4(stage)), &tm_a4, g * (KS / 2), m0, full, pol);
              tma_load_2d_hint(smem_u32(b4(stage)), &tm_b4, g * (KS / 2), nb, full, pol);
              bulk_load(smem_u32(scl(stage)), p.act_scales + (size_t)g * p.M_pad + m0, 256, full);
              bulk_load(smem_u32(scl(stage)) + 256, p.w_scales + (size_t)g * p.N_pad + nb, 256, full);
            }
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
      if (lane == 0) {
        volatile int never = 0;
        WaitCtx drain_ctx{&never, p.dev_status, kDrainLimitNs};
        for (int s = 0; s < STAGES; ++s)
          if (issued_mask & (1u << s))
            mbar_wait(smem_u32(&ctl->raw_full[s]), (issued_phase >> s) & 1, drain_ctx, kDevTimeoutDrain);
      }
    } else if (warp == MMA_WARP) {
      // ------------------------------------------------------------ MMA issuer (CTA 0)
      if (rank == 0) {
        int stage = 0;
        uint32_t phase = 0, acc_phase = 0;
        bool ok = true;
        for (int tile = pair; tile < num_tiles && ok; tile += num_pairs) {
          if (!mbar_wait_warp(smem_u32(&ctl->acc_empty), acc_phase ^ 1, wctx, kDevTimeoutMma)) {
            ok = false;
            break;
          }
          tc_fence_after();
          for (int kt = 0; kt < slices; ++kt) {
            if (!mbar_wait_warp(smem_u32(&ctl->opnd_full[stage]), phase, wctx, kDevTimeoutMma)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t sa = smem_u32(a16(stage)), sb = smem_u32(b16(stage));
            const bool leader = elect_one();
            if (leader) {
              const uint32_t idesc = kt == 0 ? IDESC_BF16 : IDESC_F16;
#pragma unroll
              for (int j = 0; j < 4; ++j)
                mma_bf16_pair(tmem, sw128_desc(sa + 32 * j), sw128_desc(sb + 32 * j), idesc,
                              (kt == 0 && j == 0) ? 0u : 1u);
              tc_commit_pair_mc(smem_u32(&ctl->empty[stage]), PAIR_MASK);
            }
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
        if (elect_one()) tc_commit_pair(smem_u32(&ctl->drain));
        __syncwarp();
        volatile int never = 0;
        WaitCtx drain_ctx{&never, p.dev_status, kDrainLimitNs};
        mbar_wait(smem_u32(&ctl->drain), 0, drain_ctx, kDevTimeoutDrain);
      }
    } else if (warp >= DQ_WARP0) {
      // ------------------------------------------------------------ dequantization
      const int t = threadIdx.x - DQ_WARP0 * 32;   // row t of A and of this CTA's half of B
      const uint32_t opnd_local = smem_u32(&ctl->opnd_full[0]);
      const uint32_t opnd_leader = rank == 0 ? opnd_local : mapa_shared(opnd_local, 0);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = pair; tile < num_tiles && ok; tile += num_pairs) {
        const int m0 = tile_m0(tile);
        const int nb = tile_n0(tile) + (int)rank * BN_HALF;
        // 2^-E of the two rows (exact reciprocals of powers of two); rows
        // past M or N have zero codes and scales, and get factor 0.
        const float inv_a = m0 + t < p.M ? __frcp_rn(__ldg(p.row_factor + m0 + t)) : 0.f;
        const float inv_b = nb + t < p.N ? __frcp_rn(__ldg(p.col_factor + nb + t)) : 0.f;
        for (int kt = 0; kt < slices; ++kt) {
          const bool got = mbar_wait(smem_u32(&ctl->raw_full[stage]), phase, wctx, kDevTimeoutMma);
          if (named_bar_any(1, DQ_THREADS, !got || ctl->abort_flag != 0)) {
            ok = false;
            break;
          }
          if (kt > 0) {
            const uint32_t sc = smem_u32(scl(stage));
            const float sa = __uint_as_float(lds_u16(sc + 2 * t) << 16);
            const float sb = __uint_as_float(lds_u16(sc + 256 + 2 * t) << 16);
            dequant_row(smem_u32(a4(stage)) + 32 * t, i4_f16x2_dup(__fmul_rn(sa, inv_a)), smem_u32(a16(stage)), t);
            dequant_row(smem_u32(b4(stage)) + 32 * t, i4_f16x2_dup(__fmul_rn(sb, inv_b)), smem_u32(b16(stage)), t);
            // The generic-proxy writes, before the tensor core reads them.
            fence_proxy_async_smem();
          }
          named_bar_sync(1, DQ_THREADS);
          if (t == 0) {
            const uint32_t bar = opnd_leader + (uint32_t)stage * 8u;
            if (rank == 0)
              mbar_arrive(bar);
            else
              mbar_arrive_cluster_release(bar);
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(EPI_REGS));
    // -------------------------------------------------------------- epilogue (both CTAs)
    // Warp w owns 32 rows (TMEM lane quarter w % 4) x 128 columns (half
    // w / 4) of this CTA's 128 x 256 accumulator: four TMEM loads and one
    // wait, the accumulator released, then y = bf16(D f_a f_w + bias)
    // through 16-column TMA stores.
    const int q = warp & 3, h = warp >> 2;
    uint8_t* buf0 = epi_base + warp * 2 * EPI_BUF_BYTES;
    const uint32_t acc_empty_local = smem_u32(&ctl->acc_empty);
    const uint32_t acc_empty_leader = rank == 0 ? acc_empty_local : mapa_shared(acc_empty_local, 0);
    const uint32_t acc_base = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(h * EPI_COLS);
    uint32_t acc_phase = 0;
    int chunk_seq = 0;
    for (int tile = pair; tile < num_tiles; tile += num_pairs) {
      const int m0 = tile_m0(tile);
      const int nw = tile_n0(tile) + h * EPI_COLS;   // this warp's first column
      const int row = m0 + 32 * q + lane;
      uint2 bias4 = make_uint2(0, 0);
      float4 f_col4 = make_float4(0.f, 0.f, 0.f, 0.f);
      if (nw + 4 * lane < p.N) {
        if (p.bias != nullptr) bias4 = __ldg(reinterpret_cast<const uint2*>(p.bias + nw) + lane);
        f_col4 = __ldg(reinterpret_cast<const float4*>(p.col_factor + nw) + lane);
      }
      const float f_row = row < p.M ? __ldg(p.row_factor + row) : 0.f;
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
        for (int hh = 0; hh < 2; ++hh) {
          const int c0 = 32 * i + EPI_CHUNK * hh;
          const int ncol = nw + c0;
          uint32_t bw[8];
          float fc[16];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int src = c0 / 4 + j;
            bw[2 * j] = __shfl_sync(0xffffffffu, bias4.x, src);
            bw[2 * j + 1] = __shfl_sync(0xffffffffu, bias4.y, src);
            // f_a f_w is a power of two: the fma below rounds once.
            fc[4 * j] = __fmul_rn(f_row, __shfl_sync(0xffffffffu, f_col4.x, src));
            fc[4 * j + 1] = __fmul_rn(f_row, __shfl_sync(0xffffffffu, f_col4.y, src));
            fc[4 * j + 2] = __fmul_rn(f_row, __shfl_sync(0xffffffffu, f_col4.z, src));
            fc[4 * j + 3] = __fmul_rn(f_row, __shfl_sync(0xffffffffu, f_col4.w, src));
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
          uint8_t* rowp = buf + lane * 32;
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const int pj = j ^ ((lane >> 2) & 1);  // 32-byte swizzle
            *reinterpret_cast<uint4*>(rowp + pj * 16) =
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
  // CTA 1's dequantization warps arrive on CTA 0's barriers.
  __syncwarp();
  tc_fence_before();
  cluster_sync();
  if (warp == MMA_WARP) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, TMEM_COLS);
  }
}

}  // namespace

cudaError_t launch_gemm_int4_pair(const GemmInt4DqParams& p, const GemmInt4DqTmaps& t, cudaStream_t stream,
                                  bool pdl) {
  static int max_pairs = -1;
  if (max_pairs < 0) {
    cudaError_t e =
        cudaFuncSetAttribute(gemm_int4_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    // setmaxnreg.inc waits until the other warpgroups have released enough
    // registers: only launch if the compiled register count makes the split
    // add up.
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, gemm_int4_pair_kernel);
    if (e != cudaSuccess) return e;
    if (fa.numRegs * NUM_THREADS < 256 * EPI_REGS + 256 * CTL_REGS) return cudaErrorInvalidConfiguration;
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
    e = cudaOccupancyMaxActiveClusters(&n, gemm_int4_pair_kernel, &q);
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
  return cudaLaunchKernelEx(&cfg, gemm_int4_pair_kernel, t.a4, t.b4, t.la, t.lb, t.y, p);
}

}  // namespace svdq
