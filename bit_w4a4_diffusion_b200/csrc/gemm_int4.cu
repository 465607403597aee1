// S3: the W4A4 INT4 GEMM (signed int4, a bf16 scale per 64 along K) with the
// low-rank up-projection and bias, on 5th-generation tensor cores.
//
// Pages: "Nunchaku Lite" docs, "Supported quantization types" table
// (svdq_w4a4, int4, group 64) and its tip that int4 checkpoints on Blackwell
// may be slower than nvfp4; "Hugging Face integrates Nunchaku 4-bit diffusion
// inference into Diffusers", section "SVDQuant and the Nunchaku engine".
//
//   P_g[m,n] = sum_{k in group g} qa[m,k] qw[n,k]             (tcgen05 kind::i8, exact int32)
//   y[m,n]   = bf16( sum_g sa[m,g] sw[n,g] P_g[m,n]            (fp32, in the epilogue)
//                    + [hi(u)|lo(u)] . [L2^T|L2^T]               (kind::f16, TMEM fp32)
//                    + bias[n] )
//
// Every 64-group needs its own rescale, so each group's int32 partial lands
// in its own TMEM buffer (four, in turn; the tile's low-rank result takes the
// first one and starts the accumulator) and the epilogue warps fold it into
// fp32 registers while the tensor core computes the next groups: the epilogue
// ALU work is what bounds this kernel (the reason the docs expect int4 to be
// slower than nvfp4 on Blackwell).  Two devices keep that work to two packed
// FMAs per pair of elements:
//  - a partial buffer is preset (tcgen05.st) to the int32 pattern of the
//    float C = 1.5 * 2^23 before its group's MMAs accumulate onto it, so the
//    exact sum P (|P| <= 64 * 7 * 7 < 2^22) comes out as the bits of the
//    float C + P: no integer-to-float conversion;
//  - the unpack warps stage each group's scales in fp32 together with
//    -s_w * C (exact: an 8-bit significand times 1.5 * 2^23), so that
//    fl(s_w * f - s_w * C) = fl(s_w * P) with f = C + P, and then
//    acc = fl(s_a * that + acc), as before.
//
// Structure: persistent CTAs, 128x128 output tiles, 14 warps:
//   warp 0      producer: TMA of the packed int4 codes and bulk copies of the
//               group scales into a 4-stage ring of K=128 slices; for the
//               low-rank slice TMA of u' and [L2^T|L2^T] straight into the
//               int8 operand buffers
//   warp 1      tcgen05 issuer
//   warps 2-5   unpack: int4 -> int8 into the SWIZZLE_128B K-major operand
//   warps 6-13  epilogue: two warps per TMEM lane quarter, 64 columns each
// All waits are bounded (see ptx.cuh); on timeout the kernel records a status,
// drains its copies and MMAs, frees TMEM and returns.
#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"
#include "svdq_internal.h"

namespace svdq {
namespace {

constexpr int BM = 128, BN = 128;
constexpr int KS = 128;                      // K elements per slice (two groups)
constexpr int STAGES = 4;
constexpr int A4_BYTES = BM * KS / 2;        // 8 KB packed int4
constexpr int B4_BYTES = BN * KS / 2;        // 8 KB
constexpr int A8_BYTES = BM * KS;            // 16 KB int8 (also u' bf16 [128 x 64])
constexpr int B8_BYTES = BN * KS;            // 16 KB int8 (also [L2^T|L2^T] bf16 [128 x 64])
constexpr int SC_BYTES = 2 * (BM + BN) * 2;  // bf16 scales of two groups, A then B
constexpr int SCF_BYTES = 2 * (BM + 2 * BN) * 4;   // fp32 of two groups: s_a [128], s_w [128], -s_w C [128]
constexpr int STAGE_BYTES = A8_BYTES + B8_BYTES + A4_BYTES + B4_BYTES + 1024 + SCF_BYTES;  // bf16 scales in 1 KB
static_assert(STAGE_BYTES % 1024 == 0, "stages keep the 1024-byte alignment of SWIZZLE_128B");
constexpr uint32_t kPresetBits = 0x4B400000u;    // the float 1.5 * 2^23 (ulp 1 over [2^23, 2^24))
constexpr float kPreset = 12582912.0f;
constexpr int UNPACK_WARPS = 4, EPI_WARPS = 8;
constexpr int EPI_COLS = 4 * BN / EPI_WARPS;   // columns per epilogue warp (4 warps per lane quarter)
constexpr int NUM_THREADS = (2 + UNPACK_WARPS + EPI_WARPS) * 32;
constexpr int TMEM_COLS = 512;
// Four partial buffers of 128 columns (all of TMEM), used in turn by the
// tile's low-rank result (fp32, the tile's first "group") and its 64-groups
// (int32 on the preset C): the MMA can run up to three groups ahead of the
// epilogue.
constexpr int NPART = 4;
constexpr int TMEM_PART = 0;
constexpr unsigned long long kDrainLimitNs = 2000000000ull;

struct SmemCtl {
  uint64_t full[STAGES];     // producer -> unpack (int4 + scales landed)
  uint64_t opnd[STAGES];     // unpack / TMA -> MMA (int8 or bf16 operands ready)
  uint64_t empty[STAGES];    // MMA commit + epilogue warps -> producer
  uint64_t part_full[NPART];    // MMA -> epilogue (group partial ready)
  uint64_t part_empty[NPART];   // epilogue -> MMA (buffer drained and preset)
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

constexpr size_t SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + sizeof(SmemCtl);

// kind::i8: s32 accumulate (c_format 2 at bit 4), signed a/b (1 at bits 7/10).
constexpr uint32_t IDESC_I8 = (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                              ((uint32_t)(BM >> 4) << 24);
constexpr uint32_t IDESC_BF16 = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                                ((uint32_t)(BM >> 4) << 24);

SVDQ_DEV uint64_t sw128_desc(uint32_t saddr) { return smem_desc(saddr, 16, 1024, 2); }

SVDQ_DEV float4 ld_shared_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr)
               : "memory");
  return v;
}


// Eight packed int4 (two's complement, element 2j in the low nibble of byte
// j) -> eight int8 in element order (two 32-bit words).
SVDQ_DEV void unpack_int4x8(uint32_t w, uint32_t& lo_out, uint32_t& hi_out) {
  uint32_t lo = w & 0x0F0F0F0Fu, hi = (w >> 4) & 0x0F0F0F0Fu;
  lo |= (lo & 0x08080808u) * 0x1Eu;  // sign-extend: 0x08 -> 0xF0 in each byte
  hi |= (hi & 0x08080808u) * 0x1Eu;
  lo_out = __byte_perm(lo, hi, 0x5140);  // e0 e1 e2 e3
  hi_out = __byte_perm(lo, hi, 0x7362);  // e4 e5 e6 e7
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
    gemm_int4_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                     const __grid_constant__ CUtensorMap tm_la, const __grid_constant__ CUtensorMap tm_lb,
                     const GemmInt4Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  SmemCtl* ctl = reinterpret_cast<SmemCtl*>(smem + STAGES * STAGE_BYTES);
  auto a8 = [&](int s) { return smem + s * STAGE_BYTES; };
  auto b8 = [&](int s) { return smem + s * STAGE_BYTES + A8_BYTES; };
  auto a4 = [&](int s) { return smem + s * STAGE_BYTES + A8_BYTES + B8_BYTES; };
  auto b4 = [&](int s) { return smem + s * STAGE_BYTES + A8_BYTES + B8_BYTES + A4_BYTES; };
  auto scl = [&](int s) {
    return reinterpret_cast<uint16_t*>(smem + s * STAGE_BYTES + A8_BYTES + B8_BYTES + A4_BYTES + B4_BYTES);
  };
  // fp32 scales of the stage's two groups: [h][s_a 128 | s_w 128 | -s_w C 128].
  auto scf = [&](int s) {
    return reinterpret_cast<float*>(smem + s * STAGE_BYTES + A8_BYTES + B8_BYTES + A4_BYTES + B4_BYTES + 1024);
  };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles_m = (p.M + BM - 1) / BM;
  const int tiles_n = (p.N + BN - 1) / BN;
  const int num_tiles = tiles_m * tiles_n;
  const int k_slices = p.K / KS;
  const int slices = k_slices + 1;  // slot 0 of every tile: the low-rank slice

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&ctl->full[s]), 1);
      mbar_init(smem_u32(&ctl->opnd[s]), 1);
      mbar_init(smem_u32(&ctl->empty[s]), 1 + EPI_WARPS);
    }
    for (int b = 0; b < NPART; ++b) {
      mbar_init(smem_u32(&ctl->part_full[b]), 1);
      mbar_init(smem_u32(&ctl->part_empty[b]), EPI_WARPS);
    }
    mbar_init(smem_u32(&ctl->drain), 1);
    ctl->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_a);
    prefetch_tmap(&tm_b);
    prefetch_tmap(&tm_la);
    prefetch_tmap(&tm_lb);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&ctl->tmem_base), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;
  pdl_wait();
  // The next kernel on the stream may be scheduled from now on; it waits for
  // this grid's completion before it reads anything.
  pdl_launch_dependents();
  WaitCtx wctx{&ctl->abort_flag, p.dev_status, p.timeout_ns};
  const size_t mpad = (size_t)p.M_pad, npad = (size_t)p.N_pad;

  // The producer and MMA loops run on whole warps and issue from one elected
  // lane (the lowest, every time): TMA and tcgen05 instructions take
  // uniform-register operands, which a loop run by lane 0 alone does not
  // keep, and each issue then costs several times more.
  if (warp == 0) {
    {
      // ------------------------------------------------------------ producer
      int stage = 0;
      // Per stage, the last use: issued (bit), its ring parity, and whether it
      // was a low-rank slice (TMA into the operand buffers, completes opnd[])
      // or a k-slice (TMA of packed codes, completes full[]).
      uint32_t phase = 0, issued_mask = 0, issued_phase = 0, lr_mask = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const int m0 = (tile % tiles_m) * BM, n0 = (tile / tiles_m) * BN;
        for (int kt = 0; kt < slices; ++kt) {
          if (!mbar_wait_warp(smem_u32(&ctl->empty[stage]), phase ^ 1, wctx, kDevTimeoutProducer)) {
            ok = false;
            break;
          }
          const bool leader = elect_one();
          if (kt == 0) {
            if (leader) {
              // full[] completes once per use of a stage, whatever the slice
              // kind, so that every waiter's parity follows the ring phase.
              mbar_arrive(smem_u32(&ctl->full[stage]));
              const uint32_t bar = smem_u32(&ctl->opnd[stage]);
              mbar_arrive_expect_tx(bar, A8_BYTES + B8_BYTES);
              tma_load_2d(smem_u32(a8(stage)), &tm_la, 0, m0, bar);
              tma_load_2d(smem_u32(b8(stage)), &tm_lb, 0, n0, bar);
            }
            lr_mask |= 1u << stage;
          } else {
            if (leader) {
              const int g0 = (kt - 1) * 2;  // first 64-group of the slice
              const uint32_t bar = smem_u32(&ctl->full[stage]);
              mbar_arrive_expect_tx(bar, A4_BYTES + B4_BYTES + SC_BYTES);
              tma_load_2d(smem_u32(a4(stage)), &tm_a, (kt - 1) * (KS / 2), m0, bar);
              tma_load_2d(smem_u32(b4(stage)), &tm_b, (kt - 1) * (KS / 2), n0, bar);
              uint16_t* sc = scl(stage);
              for (int h = 0; h < 2; ++h) {
                bulk_load(smem_u32(sc + h * BM), p.act_scales + (size_t)(g0 + h) * mpad + m0, BM * 2, bar);
                bulk_load(smem_u32(sc + 2 * BM + h * BN), p.w_scales + (size_t)(g0 + h) * npad + n0, BN * 2, bar);
              }
            }
            lr_mask &= ~(1u << stage);
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
      volatile int never = 0;
      WaitCtx drain_ctx{&never, p.dev_status, kDrainLimitNs};
      // Earlier uses of a stage were consumed before it was refilled; only the
      // last use can still have a copy in flight.
      for (int s = 0; s < STAGES; ++s) {
        if (!(issued_mask & (1u << s))) continue;
        const uint64_t* bar = (lr_mask & (1u << s)) ? &ctl->opnd[s] : &ctl->full[s];
        mbar_wait(smem_u32(bar), (issued_phase >> s) & 1, drain_ctx, kDevTimeoutDrain);
      }
    }
  } else if (warp == 1) {
    {
      // ------------------------------------------------------------ MMA issuer
      int stage = 0;
      uint32_t phase = 0;
      uint32_t pcount = 0;  // partial-buffer uses so far (low-rank results and groups)
      bool ok = true;
      // Use pcount / NPART of buffer pcount % NPART: the epilogue has drained
      // its previous use and preset it.
      auto take_part = [&]() -> bool {
        const bool got = mbar_wait_warp(smem_u32(&ctl->part_empty[pcount % NPART]), (pcount / NPART) & 1, wctx,
                                        kDevTimeoutMma);
        tc_fence_after();
        return got;
      };
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        for (int kt = 0; kt < slices && ok; ++kt) {
          if (!mbar_wait_warp(smem_u32(&ctl->opnd[stage]), phase, wctx, kDevTimeoutMma)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(a8(stage)), sb = smem_u32(b8(stage));
          if (kt == 0) {
            // The low-rank result (fp32, overwriting the preset).
            if (!take_part()) {
              ok = false;
              break;
            }
            const uint32_t d = tmem + TMEM_PART + (pcount % NPART) * BN;
            if (elect_one()) {
#pragma unroll
              for (int j = 0; j < 4; ++j)
                mma_bf16(d, sw128_desc(sa + 32 * j), sw128_desc(sb + 32 * j), IDESC_BF16, j > 0 ? 1u : 0u);
              tc_commit(smem_u32(&ctl->part_full[pcount % NPART]));
            }
            __syncwarp();
            ++pcount;
          } else {
            for (int h = 0; h < 2; ++h, ++pcount) {
              const int pb = pcount % NPART;
              if (!take_part()) {
                ok = false;
                break;
              }
              const uint32_t d = tmem + TMEM_PART + pb * BN;
              if (elect_one()) {
                mma_i8(d, sw128_desc(sa + 64 * h), sw128_desc(sb + 64 * h), IDESC_I8, 1u);
                mma_i8(d, sw128_desc(sa + 64 * h + 32), sw128_desc(sb + 64 * h + 32), IDESC_I8, 1u);
                tc_commit(smem_u32(&ctl->part_full[pb]));
              }
              __syncwarp();
            }
            if (!ok) break;
          }
          if (elect_one()) tc_commit(smem_u32(&ctl->empty[stage]));
          __syncwarp();
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // Every MMA the elected lane issued completes before TMEM is freed.
      if (elect_one()) tc_commit(smem_u32(&ctl->drain));
      __syncwarp();
      volatile int never = 0;
      WaitCtx drain_ctx{&never, p.dev_status, kDrainLimitNs};
      mbar_wait(smem_u32(&ctl->drain), 0, drain_ctx, kDevTimeoutDrain);
    }
  } else if (warp < 2 + UNPACK_WARPS) {
    // -------------------------------------------------------------- unpack
    const int t = threadIdx.x - 64;  // 0..127: one A row and one B row per slice
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
      for (int kt = 0; kt < slices; ++kt) {
        if (kt > 0) {
          const bool got = mbar_wait(smem_u32(&ctl->full[stage]), phase, wctx, kDevTimeoutMma);
          if (!__all_sync(0xffffffffu, got)) {
            ok = false;
          }
          // all 128 unpack threads take the same branch: the abort flag is shared
          if (ok) {
            // 16-byte piece i = t + 128 j of the 8 KB packed tile is row i / 4,
            // columns 32 (i % 4) .. + 31: a warp reads 512 contiguous bytes
            // (no bank conflict; one thread per 64-byte row made every
            // quarter-warp load hit two bank groups), and the two 16-byte
            // int8 chunks it writes land, under the 128-byte swizzle, in
            // chunk sets of opposite parity for the two rows of a
            // quarter-warp (no conflict either).
            for (int op = 0; op < 2; ++op) {
              const uint8_t* src = op == 0 ? a4(stage) : b4(stage);
              uint8_t* dst = op == 0 ? a8(stage) : b8(stage);
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const int i = t + 128 * j;
                const int r = i >> 2, c = i & 3;
                const uint4 w = *reinterpret_cast<const uint4*>(src + 16 * i);
                uint4 o0, o1;
                unpack_int4x8(w.x, o0.x, o0.y);
                unpack_int4x8(w.y, o0.z, o0.w);
                unpack_int4x8(w.z, o1.x, o1.y);
                unpack_int4x8(w.w, o1.z, o1.w);
                uint8_t* row = dst + r * KS;
                *reinterpret_cast<uint4*>(row + 16 * ((2 * c) ^ (r & 7))) = o0;
                *reinterpret_cast<uint4*>(row + 16 * ((2 * c + 1) ^ (r & 7))) = o1;
              }
            }
            fence_proxy_async_smem();
            // The epilogue's fp32 scales of both groups: row t of A, column t of B.
            const uint16_t* sc = scl(stage);
            float* sf = scf(stage);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const float sw = __bfloat162float(__ushort_as_bfloat16(sc[2 * BM + h * BN + t]));
              sf[h * (BM + 2 * BN) + t] = __bfloat162float(__ushort_as_bfloat16(sc[h * BM + t]));
              sf[h * (BM + 2 * BN) + BM + t] = sw;
              sf[h * (BM + 2 * BN) + BM + BN + t] = __fmul_rn(sw, -kPreset);   // exact
            }
          }
          // The stop decision is taken inside the barrier (an OR over all
          // unpack threads), so that no unpack warp can go on to the next
          // barrier after another one has left.
          if (named_bar_any(1, UNPACK_WARPS * 32, !ok || ctl->abort_flag != 0)) {
            ok = false;
            break;
          }
          if (threadIdx.x == 64) mbar_arrive(smem_u32(&ctl->opnd[stage]));
        }
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
  } else {
    // -------------------------------------------------------------- epilogue
    const int e = warp - (2 + UNPACK_WARPS);  // 0 .. EPI_WARPS - 1
    const int q = warp & 3;                   // TMEM lane quarter
    const int ch = e >> 2;                    // column block of EPI_COLS
    const int row = 32 * q + lane;            // row of the tile this thread owns
    int stage = 0;
    uint32_t phase = 0, pcount = 0;
    bool ok = true;
    // This warp's columns of partial buffer pb.
    auto part_addr = [&](int pb) {
      return tmem + ((uint32_t)(32 * q) << 16) + TMEM_PART + pb * BN + EPI_COLS * ch;
    };
    // Preset this warp's columns of buffer pb to C and hand it to the MMA warp.
    auto preset_release = [&](int pb) {
      const uint32_t a = part_addr(pb);
#pragma unroll
      for (int c8 = 0; c8 < EPI_COLS / 8; ++c8) tmem_st_32x32b_x8_fill(a + 8 * c8, kPresetBits);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&ctl->part_empty[pb]));
    };
#pragma unroll
    for (int b = 0; b < NPART; ++b) preset_release(b);
    auto wait_part = [&](int pb) -> bool {
      const bool got = mbar_wait(smem_u32(&ctl->part_full[pb]), (pcount / NPART) & 1, wctx, kDevTimeoutEpilogue);
      if (!__all_sync(0xffffffffu, got)) return false;
      tc_fence_after();
      return true;
    };
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
      const int m0 = (tile % tiles_m) * BM, n0 = (tile / tiles_m) * BN;
      float2 acc[EPI_COLS / 2];   // columns (2 i, 2 i + 1) of this thread's EPI_COLS
      for (int kt = 0; kt < slices && ok; ++kt) {
        if (kt == 0) {
          // The low-rank result starts the accumulator.
          const int pb = pcount % NPART;
          if (!wait_part(pb)) {
            ok = false;
            break;
          }
          const uint32_t taddr = part_addr(pb);
#pragma unroll
          for (int qc = 0; qc < EPI_COLS / 16; ++qc) {
            uint32_t r[16];
            tmem_ld_32x32b_x16(taddr + 16 * qc, r);
            tmem_ld_wait(r);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              acc[8 * qc + i] = make_float2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
          }
          preset_release(pb);
          ++pcount;
        } else {
          // The slice's fp32 scales, staged by the unpack warps.
          const bool sc_ok = mbar_wait(smem_u32(&ctl->opnd[stage]), phase, wctx, kDevTimeoutEpilogue);
          if (!__all_sync(0xffffffffu, sc_ok)) {
            ok = false;
            break;
          }
          const float* sf = scf(stage);
          for (int h = 0; h < 2; ++h, ++pcount) {
            const int pb = pcount % NPART;
            if (!wait_part(pb)) {
              ok = false;
              break;
            }
            const float* sfh = sf + h * (BM + 2 * BN);
            const float sa1 = sfh[row];
            const float2 sa = make_float2(sa1, sa1);
            const float* swp = sfh + BM + EPI_COLS * ch;     // s_w of this warp's columns
            const float* ncp = swp + BN;                     // -s_w C
            const uint32_t taddr = part_addr(pb);
            // 16 columns per TMEM load (a 32-column block and its sixteen
            // scale vectors would not fit beside the accumulator).
#pragma unroll
            for (int qc = 0; qc < EPI_COLS / 16; ++qc) {
              uint32_t r[16];
              tmem_ld_32x32b_x16(taddr + 16 * qc, r);
              tmem_ld_wait(r);
              if (qc == EPI_COLS / 16 - 1) preset_release(pb);   // every column is in registers
#pragma unroll
              for (int v = 0; v < 4; ++v) {
                const float4 w4 = ld_shared_f4(smem_u32(swp + 16 * qc + 4 * v));
                const float4 n4 = ld_shared_f4(smem_u32(ncp + 16 * qc + 4 * v));
                // r holds the bits of C + P: fl(s_w (C + P) - s_w C) = fl(s_w P).
                const float2 t0 = __ffma2_rn(make_float2(w4.x, w4.y),
                                             make_float2(__uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1])),
                                             make_float2(n4.x, n4.y));
                const float2 t1 = __ffma2_rn(make_float2(w4.z, w4.w),
                                             make_float2(__uint_as_float(r[4 * v + 2]), __uint_as_float(r[4 * v + 3])),
                                             make_float2(n4.z, n4.w));
                const int j = 8 * qc + 2 * v;
                acc[j] = __ffma2_rn(sa, t0, acc[j]);
                acc[j + 1] = __ffma2_rn(sa, t1, acc[j + 1]);
              }
            }
          }
          if (!ok) break;
        }
        // Every slice of the ring is released by the MMA commit and all eight
        // epilogue warps (they read the scales held in the slice).
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&ctl->empty[stage]));
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (!ok) break;
      // y = bf16(acc + bias): the low-rank result is already in acc.
      const int m = m0 + row;
#pragma unroll
      for (int qc = 0; qc < EPI_COLS / 16; ++qc) {
        const int nb = n0 + EPI_COLS * ch + 16 * qc;
        if (m < p.M && nb < p.N) {
          uint16_t* yrow = p.y + (size_t)m * p.N + nb;
#pragma unroll
          for (int v = 0; v < 2; ++v) {
            uint32_t pk[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int j = 8 * v + 2 * i;
              float y0 = acc[8 * qc + j / 2].x, y1 = acc[8 * qc + j / 2].y;
              if (p.bias) {
                y0 = __fadd_rn(y0, __bfloat162float(__ushort_as_bfloat16(p.bias[nb + j])));
                y1 = __fadd_rn(y1, __bfloat162float(__ushort_as_bfloat16(p.bias[nb + j + 1])));
              }
              __nv_bfloat162 hh = __floats2bfloat162_rn(y0, y1);
              pk[i] = *reinterpret_cast<uint32_t*>(&hh);
            }
            *reinterpret_cast<uint4*>(yrow + 8 * v) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace

cudaError_t launch_gemm_int4(const GemmInt4Params& p, const GemmInt4Tmaps& t, int num_sms, cudaStream_t stream,
                             bool pdl) {
  cudaError_t e = cudaFuncSetAttribute(gemm_int4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
  if (e != cudaSuccess) return e;
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
  return cudaLaunchKernelEx(&cfg, gemm_int4_kernel, t.a, t.b, t.la, t.lb, p);
}

}  // namespace svdq
