// Host-side (untimed) weight preparation for the W4A4 and W4A16 layers, and
// the NVFP4 scale-layout helpers.  Built with -ffp-contract=off: every fp32
// step below is one IEEE operation.
//
// Page: "Hugging Face integrates Nunchaku 4-bit diffusion inference into
// Diffusers", section "SVDQuant and the Nunchaku engine" (outliers migrate to
// the weights, a 16-bit low-rank branch absorbs the hard part, the residual is
// quantized to 4 bits); "Nunchaku Lite" docs, "Supported quantization types"
// table (nvfp4 group 16, int4 group 64, awq_w4a16 int4 group 64).
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

#include "svdq.h"

namespace {

float bf16_to_f32(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

uint16_t f32_to_bf16_rne(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  const uint32_t lsb = (u >> 16) & 1u;
  return (uint16_t)((u + 0x7FFFu + lsb) >> 16);  // finite inputs only
}

// Finite fp32 with |v| <= 65504 -> fp16 bits, round to nearest even (the
// subnormal range included).
uint16_t f32_to_f16_rne(float v) {
  uint32_t u;
  std::memcpy(&u, &v, 4);
  const uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
  const float a = std::fabs(v);
  if (a == 0.0f) return sign;
  int e;
  std::frexp(a, &e);  // a = m * 2^e, m in [0.5, 1)
  // Quantum of the fp16 grid at a: 2^(e-11) for normals, 2^-24 in the subnormal range.
  const int qexp = std::max(e - 11, -24);
  const float q = std::nearbyint(std::ldexp(a, -qexp));  // integer significand, RNE
  const float r = std::ldexp(q, qexp);                     // rounded value, exact in fp32
  if (r < 6.103515625e-05f) return (uint16_t)(sign | (uint16_t)std::ldexp(r, 24));  // subnormal
  int re;
  const float rm = std::frexp(r, &re);                     // r = rm * 2^re
  const uint32_t mant = (uint32_t)std::ldexp(rm, 11) - 1024u;  // 10 stored bits
  return (uint16_t)(sign | ((uint32_t)(re - 1 + 15) << 10) | mant);
}

// Non-negative finite fp32 -> E4M3 byte, round to nearest even, saturating at
// 448 (0x7E).  Works on the fp32 fields directly.
uint8_t e4m3_rne_sat(float t) {
  if (!(t > 0.f)) return 0;
  if (t >= 448.f) return 0x7E;
  uint32_t u;
  std::memcpy(&u, &t, 4);
  const int e = (int)((u >> 23) & 0xFF) - 127;
  if (e < -6) {
    // Subnormal range of E4M3: value = m * 2^-9, m = rne(t * 2^9) in [0, 8];
    // m == 8 is the smallest normal 2^-6, whose code is also 8.
    return (uint8_t)std::nearbyint(t * 512.0f);
  }
  uint32_t m3 = (u >> 20) & 7u;
  const uint32_t rem = u & 0xFFFFFu;
  if (rem > 0x80000u || (rem == 0x80000u && (m3 & 1u))) ++m3;
  int ee = e;
  if (m3 == 8) {
    m3 = 0;
    ++ee;
  }
  const uint32_t code = ((uint32_t)(ee + 7) << 3) | m3;
  return (uint8_t)std::min<uint32_t>(code, 0x7E);
}

float e4m3_to_f32(uint8_t b) {
  const int e = (b >> 3) & 0xF, m = b & 7;
  if (e == 0) return std::ldexp((float)m, -9);
  return std::ldexp((float)(8 + m), e - 10);
}

// fp32 -> E2M1 code (sign in bit 3), round to nearest even on the grid
// {0, .5, 1, 1.5, 2, 3, 4, 6}, saturating at 6.  Midpoints are decided by
// which side holds the even code.
uint8_t e2m1_rne_sat(float v) {
  const uint8_t s = std::signbit(v) ? 8 : 0;
  const float a = std::fabs(v);
  uint8_t c;
  if (a <= 0.25f) c = 0;
  else if (a < 0.75f) c = 1;
  else if (a <= 1.25f) c = 2;
  else if (a < 1.75f) c = 3;
  else if (a <= 2.5f) c = 4;
  else if (a < 3.5f) c = 5;
  else if (a <= 5.0f) c = 6;
  else c = 7;
  return (uint8_t)(s | c);
}

template <class F>
void parallel_rows(int n, F&& f) {
  unsigned nt = std::max(1u, std::min(16u, std::thread::hardware_concurrency()));
  if (n < 64) nt = 1;
  std::vector<std::thread> th;
  for (unsigned t = 0; t < nt; ++t)
    th.emplace_back([&, t] {
      for (int i = (int)t; i < n; i += (int)nt) f(i);
    });
  for (auto& x : th) x.join();
}

size_t sf_offset(int row, int group, int K) {
  return ((size_t)(row >> 7) * (K / 64) + (group >> 2)) * 512 + (row & 31) * 16 + ((row & 127) >> 5) * 4 + (group & 3);
}

}  // namespace

extern "C" {

int svdq_scales_to_rowmajor(int rows, int K, const uint8_t* tiled, uint8_t* rowmajor) {
  if (rows <= 0 || K <= 0 || K % 64 || !tiled || !rowmajor) return SVDQ_ERR_INVALID_ARG;
  for (int r = 0; r < rows; ++r)
    for (int g = 0; g < K / 16; ++g) rowmajor[(size_t)r * (K / 16) + g] = tiled[sf_offset(r, g, K)];
  return SVDQ_OK;
}

int svdq_scales_from_rowmajor(int rows, int K, const uint8_t* rowmajor, uint8_t* tiled) {
  if (rows <= 0 || K <= 0 || K % 64 || !tiled || !rowmajor) return SVDQ_ERR_INVALID_ARG;
  const int rp = (rows + 255) / 256 * 256;
  std::memset(tiled, 0, (size_t)rp * (K / 16));
  for (int r = 0; r < rows; ++r)
    for (int g = 0; g < K / 16; ++g) tiled[sf_offset(r, g, K)] = rowmajor[(size_t)r * (K / 16) + g];
  return SVDQ_OK;
}

int svdq_pack_weights(int precision, int N, int K, int rank, const uint16_t* W, const float* smooth,
                      const uint16_t* L1, const uint16_t* L2, uint8_t* codes, uint8_t* scales, float* weight_scale,
                      float* inv_smooth, uint16_t* lora_down, uint16_t* lora_up) {
  if (precision != SVDQ_NVFP4 && precision != SVDQ_INT4) return SVDQ_ERR_INVALID_ARG;
  if (N <= 0 || K <= 0 || N % 128 || K % 256 || rank != SVDQ_RANK) return SVDQ_ERR_UNSUPPORTED_SHAPE;
  if (!W || !smooth || !L1 || !L2 || !codes || !scales || !weight_scale || !inv_smooth || !lora_down || !lora_up)
    return SVDQ_ERR_INVALID_ARG;
  for (int k = 0; k < K; ++k)
    if (!(smooth[k] > 0.f) || !std::isfinite(smooth[k])) return SVDQ_ERR_INVALID_ARG;
  const int r = rank;

  for (int k = 0; k < K; ++k) inv_smooth[k] = 1.0f / smooth[k];
  // The down-projection operand: bf16 as given for INT4; for NVFP4 converted to
  // fp16 (exact for |v| in [2^-17, 65504]: bf16 has 8 significand bits).
  for (int i = 0; i < K * r; ++i)
    if (precision == SVDQ_NVFP4 && !(std::fabs(bf16_to_f32(L1[i])) <= 65504.0f)) return SVDQ_ERR_INVALID_ARG;
  for (int t = 0; t < r; ++t)
    for (int k = 0; k < K; ++k) {
      const uint16_t v = L1[(size_t)k * r + t];
      lora_down[(size_t)t * K + k] = precision == SVDQ_NVFP4 ? f32_to_f16_rne(bf16_to_f32(v)) : v;
    }
  for (int n = 0; n < N; ++n)
    for (int t = 0; t < r; ++t) {
      lora_up[(size_t)n * 2 * r + t] = L2[(size_t)t * N + n];
      lora_up[(size_t)n * 2 * r + r + t] = L2[(size_t)t * N + n];
    }

  // Residual R = fp32(W diag(lambda) - (L1 L2)^T), fp64 sum in ascending t.
  std::vector<float> R((size_t)N * K);
  std::vector<double> L1d((size_t)K * r);
  for (size_t i = 0; i < L1d.size(); ++i) L1d[i] = bf16_to_f32(L1[i]);
  parallel_rows(N, [&](int n) {
    double l2[SVDQ_RANK];
    for (int t = 0; t < r; ++t) l2[t] = bf16_to_f32(L2[(size_t)t * N + n]);
    for (int k = 0; k < K; ++k) {
      double acc = 0.0;
      const double* l1 = &L1d[(size_t)k * r];
      for (int t = 0; t < r; ++t) acc += l2[t] * l1[t];
      const double wh = (double)bf16_to_f32(W[(size_t)n * K + k]) * (double)smooth[k];
      R[(size_t)n * K + k] = (float)(wh - acc);
    }
  });

  std::memset(scales, 0, (size_t)svdq_weight_scale_bytes(precision, N, K));
  if (precision == SVDQ_NVFP4) {
    float amax = 0.f;
    for (float v : R) amax = std::max(amax, std::fabs(v));
    const float s = amax > 0.f ? amax / 2688.0f : 1.0f;
    *weight_scale = s;
    const float six_s = 6.0f * s;
    const float inv_six_s = 1.0f / six_s;
    parallel_rows(N, [&](int n) {
      const float* row = &R[(size_t)n * K];
      for (int g = 0; g < K / 16; ++g) {
        float a = 0.f;
        for (int i = 0; i < 16; ++i) a = std::max(a, std::fabs(row[16 * g + i]));
        const uint8_t sb = e4m3_rne_sat(a * inv_six_s);
        const float d = e4m3_to_f32(sb) * s;
        const float rd = d != 0.f ? 1.0f / d : 0.f;
        scales[sf_offset(n, g, K)] = sb;
        for (int i = 0; i < 16; i += 2) {
          uint8_t c0 = 0, c1 = 0;
          if (d != 0.f) {
            c0 = e2m1_rne_sat(row[16 * g + i] * rd);
            c1 = e2m1_rne_sat(row[16 * g + i + 1] * rd);
          }
          codes[(size_t)n * (K / 2) + (16 * g + i) / 2] = (uint8_t)(c0 | (c1 << 4));
        }
      }
    });
  } else {
    *weight_scale = 1.0f;
    const int np = (N + 255) / 256 * 256;
    uint16_t* sc16 = reinterpret_cast<uint16_t*>(scales);
    parallel_rows(N, [&](int n) {
      const float* row = &R[(size_t)n * K];
      for (int g = 0; g < K / 64; ++g) {
        float a = 0.f;
        for (int i = 0; i < 64; ++i) a = std::max(a, std::fabs(row[64 * g + i]));
        const uint16_t scb = f32_to_bf16_rne(a / 7.0f);
        const float sc = bf16_to_f32(scb);
        const float rs = sc != 0.f ? 1.0f / sc : 0.f;
        sc16[(size_t)g * np + n] = scb;
        for (int i = 0; i < 64; i += 2) {
          int q0 = 0, q1 = 0;
          if (sc != 0.f) {
            q0 = std::clamp((int)std::nearbyint(row[64 * g + i] * rs), -8, 7);
            q1 = std::clamp((int)std::nearbyint(row[64 * g + i + 1] * rs), -8, 7);
          }
          codes[(size_t)n * (K / 2) + (64 * g + i) / 2] = (uint8_t)((q0 & 0xF) | ((q1 & 0xF) << 4));
        }
      }
    });
  }
  return SVDQ_OK;
}

int awq_pack_weights(int N, int K, const uint16_t* W, uint8_t* qweight, uint16_t* scales, uint8_t* zeros) {
  if (N <= 0 || K <= 0 || K % 128) return SVDQ_ERR_UNSUPPORTED_SHAPE;
  if (!W || !qweight || !scales || !zeros) return SVDQ_ERR_INVALID_ARG;
  std::memset(zeros, 0, (size_t)N * (K / 128));
  parallel_rows(N, [&](int n) {
    for (int g = 0; g < K / 64; ++g) {
      const uint16_t* w = W + (size_t)n * K + 64 * g;
      float mx = bf16_to_f32(w[0]), mn = mx;
      for (int i = 1; i < 64; ++i) {
        const float v = bf16_to_f32(w[i]);
        mx = std::max(mx, v);
        mn = std::min(mn, v);
      }
      float rng = mx - mn;
      if (rng == 0.f) rng = std::fabs(mx);
      if (rng == 0.f) rng = 1.0f;
      const uint16_t scb = f32_to_bf16_rne(rng / 15.0f);
      const float sc = bf16_to_f32(scb);
      const int z = std::clamp((int)std::nearbyint(-mn / sc), 0, 15);
      scales[(size_t)n * (K / 64) + g] = scb;
      zeros[(size_t)n * (K / 128) + g / 2] |= (uint8_t)(z << (4 * (g & 1)));
      for (int i = 0; i < 64; i += 2) {
        const int q0 = std::clamp((int)std::nearbyint(bf16_to_f32(w[i]) / sc) + z, 0, 15);
        const int q1 = std::clamp((int)std::nearbyint(bf16_to_f32(w[i + 1]) / sc) + z, 0, 15);
        qweight[(size_t)n * (K / 2) + (64 * g + i) / 2] = (uint8_t)(q0 | (q1 << 4));
      }
    }
  });
  return SVDQ_OK;
}

}  // extern "C"
