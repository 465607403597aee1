// svdq_calibrate: the offline calibration that produces an svdq_w4a4 layer's
// smoothing factors, rank-r factors and static activation scale (host C++,
// fp64 for the decomposition).
//
// Page: "Hugging Face integrates Nunchaku 4-bit diffusion inference into
// Diffusers", section "SVDQuant and the Nunchaku engine": outliers migrate
// from the activations into the weights, and a 16-bit low-rank branch
// obtained by decomposing the weights absorbs their hardest part.  The
// decomposition is a randomized subspace iteration (Halko, Martinsson &
// Tropp, "Finding structure with randomness", 2011, Algorithm 4.4) with a
// caller-supplied Gaussian test matrix:
//   lambda_j = sqrt(max_i |x_ij| / max_n |W_nj|)  (fp32; 1 where a max is 0)
//   A = (W diag(lambda))^T  [K, N], never formed: products read W directly
//   Q = qr(A Omega); q times: Z = qr(A^T Q), Q = qr(A Z)
//   B = Q^T A; B B^T = Ub diag(s^2) Ub^T (cyclic Jacobi), Vt = diag(1/s) Ub^T B
//   U = Q Ub; column signs so that each column of U has its largest-magnitude
//   entry positive; L1 = bf16(U_r diag(s_r)), L2 = bf16(Vt_r)
//   s_a = max |x_ij * fp32(1/lambda_j)| / 2688
// The products A X and A^T Y are split into a fixed number of row blocks of
// W whose partial sums are added in block order, so the result does not
// depend on the number of threads.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

#include "svdq.h"
#include "svdq_internal.h"

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
  if ((u & 0x7F800000u) == 0x7F800000u) return (uint16_t)((u >> 16) | ((u & 0xFFFFu) ? 0x40u : 0u));  // inf / nan
  const uint32_t lsb = (u >> 16) & 1u;
  u += 0x7FFFu + lsb;
  return (uint16_t)(u >> 16);
}

constexpr int kBlocks = 64;  // fixed row blocks of W for the products

template <class F>
void parallel_for(int n, F&& f) {
  const int hw = std::max(1u, std::thread::hardware_concurrency());
  const int nt = std::min(n, hw);
  std::vector<std::thread> pool;
  for (int t = 0; t < nt; ++t)
    pool.emplace_back([&, t] {
      for (int i = t; i < n; i += nt) f(i);
    });
  for (auto& th : pool) th.join();
}

// The row-block kernels of the two products are compiled for AVX2 and for
// the baseline x86-64 target; the dynamic loader picks one by the host CPU.
// Both give the same bits: the host code is built without multiply-add
// contraction, and the element order of every sum is the loop order below.
#if defined(__x86_64__) && defined(__GNUC__) && !defined(__clang__)
#define SVDQ_HOST_CLONES __attribute__((target_clones("avx2", "default")))
#else
#define SVDQ_HOST_CLONES
#endif

// P [K, l] += sum over rows n0..n1-1 of W[n, k] X[n, :] (rows in order).
SVDQ_HOST_CLONES
void mul_A_block(const uint16_t* W, int K, const double* X, int l, int n0, int n1, double* P) {
  std::vector<double> wrow(K);
  for (int n = n0; n < n1; ++n) {
    for (int k = 0; k < K; ++k) wrow[k] = (double)bf16_to_f32(W[(size_t)n * K + k]);
    const double* xr = X + (size_t)n * l;
    for (int k = 0; k < K; ++k) {
      const double w = wrow[k];
      if (w == 0.0) continue;
      double* pr = P + (size_t)k * l;
      for (int c = 0; c < l; ++c) pr[c] += w * xr[c];
    }
  }
}

// Z [n, :] = sum over k of W[n, k] ly[k, :] (k in order), rows n0..n1-1.
SVDQ_HOST_CLONES
void mul_At_block(const uint16_t* W, int K, const double* ly, int l, int n0, int n1, double* Z) {
  std::vector<double> acc(l);
  for (int n = n0; n < n1; ++n) {
    std::fill(acc.begin(), acc.end(), 0.0);
    for (int k = 0; k < K; ++k) {
      const double w = (double)bf16_to_f32(W[(size_t)n * K + k]);
      if (w == 0.0) continue;
      const double* yr = ly + (size_t)k * l;
      for (int c = 0; c < l; ++c) acc[c] += w * yr[c];
    }
    std::copy(acc.begin(), acc.end(), Z + (size_t)n * l);
  }
}

// Y [K, l] = A X with A = (W diag(lam))^T, W [N, K] bf16, X [N, l].
void mul_A(const uint16_t* W, const double* lam, int N, int K, const double* X, int l, double* Y) {
  std::vector<double> part((size_t)kBlocks * K * l, 0.0);
  parallel_for(kBlocks, [&](int b) {
    const int n0 = (int)((long long)N * b / kBlocks), n1 = (int)((long long)N * (b + 1) / kBlocks);
    mul_A_block(W, K, X, l, n0, n1, part.data() + (size_t)b * K * l);
  });
  for (int k = 0; k < K; ++k)
    for (int c = 0; c < l; ++c) {
      double s = 0.0;
      for (int b = 0; b < kBlocks; ++b) s += part[((size_t)b * K + k) * l + c];
      Y[(size_t)k * l + c] = lam[k] * s;
    }
}

// Z [N, l] = A^T Y = W diag(lam) Y, Y [K, l].
void mul_At(const uint16_t* W, const double* lam, int N, int K, const double* Y, int l, double* Z) {
  std::vector<double> ly((size_t)K * l);
  for (int k = 0; k < K; ++k)
    for (int c = 0; c < l; ++c) ly[(size_t)k * l + c] = lam[k] * Y[(size_t)k * l + c];
  parallel_for(kBlocks, [&](int b) {
    const int n0 = (int)((long long)N * b / kBlocks), n1 = (int)((long long)N * (b + 1) / kBlocks);
    mul_At_block(W, K, ly.data(), l, n0, n1, Z);
  });
}

// Applies the Householder reflection I - 2 v v^T / vn (v acting on rows
// j..rows-1) to columns c0..l-1 of X [rows, l] (row-major): per column,
// d = 2 (v . x) / vn, then x -= d v.  The columns are independent, so all
// the dot products are taken in one pass over the rows and all the updates
// in a second one (contiguous rows, each column's sum still over rows in
// increasing order).
void reflect(double* X, int rows, int l, int j, int c0, const std::vector<double>& v, double vn) {
  std::vector<double> d(l - c0, 0.0);
  for (int i = j; i < rows; ++i) {
    const double vi = v[i - j];
    const double* xi = X + (size_t)i * l;
    for (int c = c0; c < l; ++c) d[c - c0] += vi * xi[c];
  }
  for (double& t : d) t = 2.0 * t / vn;
  for (int i = j; i < rows; ++i) {
    const double vi = v[i - j];
    double* xi = X + (size_t)i * l;
    for (int c = c0; c < l; ++c) xi[c] -= d[c - c0] * vi;
  }
}

void orthonormalize(double* V, int rows, int l) {
  std::vector<double> R((size_t)rows * l);
  std::copy(V, V + (size_t)rows * l, R.begin());
  std::vector<std::vector<double>> hv(l);
  for (int j = 0; j < l; ++j) {
    double norm = 0.0;
    for (int i = j; i < rows; ++i) norm += R[(size_t)i * l + j] * R[(size_t)i * l + j];
    norm = std::sqrt(norm);
    std::vector<double> v(rows - j);
    for (int i = j; i < rows; ++i) v[i - j] = R[(size_t)i * l + j];
    const double alpha = v[0] >= 0 ? -norm : norm;
    v[0] -= alpha;
    double vn = 0.0;
    for (double t : v) vn += t * t;
    if (vn > 0) reflect(R.data(), rows, l, j, j, v, vn);
    hv[j] = std::move(v);
  }
  // Q = H_0 H_1 ... H_{l-1} applied to the first l columns of the identity
  std::fill(V, V + (size_t)rows * l, 0.0);
  for (int j = 0; j < l; ++j) V[(size_t)j * l + j] = 1.0;
  for (int j = l - 1; j >= 0; --j) {
    const std::vector<double>& v = hv[j];
    double vn = 0.0;
    for (double t : v) vn += t * t;
    if (vn == 0) continue;
    reflect(V, rows, l, j, 0, v, vn);
  }
}

// Eigen-decomposition of the symmetric G [l, l] by cyclic Jacobi rotations:
// on return G's diagonal holds the eigenvalues and E [l, l] the eigenvectors
// (column c for eigenvalue c).
void jacobi_eigen(std::vector<double>& G, int l, std::vector<double>& E) {
  E.assign((size_t)l * l, 0.0);
  for (int i = 0; i < l; ++i) E[(size_t)i * l + i] = 1.0;
  for (int sweep = 0; sweep < 100; ++sweep) {
    double off = 0.0;
    for (int p = 0; p < l; ++p)
      for (int q = p + 1; q < l; ++q) off += G[(size_t)p * l + q] * G[(size_t)p * l + q];
    if (off < 1e-30) break;
    for (int p = 0; p < l; ++p)
      for (int q = p + 1; q < l; ++q) {
        const double gpq = G[(size_t)p * l + q];
        if (std::fabs(gpq) < 1e-300) continue;
        const double theta = (G[(size_t)q * l + q] - G[(size_t)p * l + p]) / (2.0 * gpq);
        const double t = (theta >= 0 ? 1.0 : -1.0) / (std::fabs(theta) + std::sqrt(theta * theta + 1.0));
        const double c = 1.0 / std::sqrt(t * t + 1.0), s = t * c;
        for (int k = 0; k < l; ++k) {  // G <- G J (columns p, q)
          const double gkp = G[(size_t)k * l + p], gkq = G[(size_t)k * l + q];
          G[(size_t)k * l + p] = c * gkp - s * gkq;
          G[(size_t)k * l + q] = s * gkp + c * gkq;
        }
        for (int k = 0; k < l; ++k) {  // G <- J^T G (rows p, q)
          const double gpk = G[(size_t)p * l + k], gqk = G[(size_t)q * l + k];
          G[(size_t)p * l + k] = c * gpk - s * gqk;
          G[(size_t)q * l + k] = s * gpk + c * gqk;
        }
        for (int k = 0; k < l; ++k) {  // E <- E J
          const double ekp = E[(size_t)k * l + p], ekq = E[(size_t)k * l + q];
          E[(size_t)k * l + p] = c * ekp - s * ekq;
          E[(size_t)k * l + q] = s * ekp + c * ekq;
        }
      }
  }
}

}  // namespace

extern "C" int svdq_calibrate(int N, int K, int M, int rank, int oversample, int power_iters, const uint16_t* W,
                              const uint16_t* x, const double* omega, float* smooth, uint16_t* L1, uint16_t* L2,
                              float* act_scale) {
  if (N <= 0 || K <= 0 || M <= 0 || rank <= 0 || oversample < 0 || power_iters < 0)
    return svdq::record_error(SVDQ_ERR_UNSUPPORTED_SHAPE, "calibrate: N=%d K=%d M=%d rank=%d oversample=%d q=%d", N,
                              K, M, rank, oversample, power_iters);
  const int l = rank + oversample;
  if (l > K || l > N)
    return svdq::record_error(SVDQ_ERR_UNSUPPORTED_SHAPE, "calibrate: rank + oversample = %d exceeds min(K, N)", l);
  if (!W || !x || !omega || !smooth || !L1 || !L2 || !act_scale)
    return svdq::record_error(SVDQ_ERR_INVALID_ARG, "calibrate: null pointer argument");

  // smoothing factors and the static activation scale (fp32, as specified)
  std::vector<float> ax(K, 0.f), aw(K, 0.f);
  for (int i = 0; i < M; ++i)
    for (int k = 0; k < K; ++k) ax[k] = std::max(ax[k], std::fabs(bf16_to_f32(x[(size_t)i * K + k])));
  for (int n = 0; n < N; ++n)
    for (int k = 0; k < K; ++k) aw[k] = std::max(aw[k], std::fabs(bf16_to_f32(W[(size_t)n * K + k])));
  std::vector<double> lam(K);
  for (int k = 0; k < K; ++k) {
    smooth[k] = (ax[k] > 0.f && aw[k] > 0.f) ? std::sqrt(ax[k] / aw[k]) : 1.0f;
    lam[k] = (double)smooth[k];
  }
  float amax = 0.f;
  for (int k = 0; k < K; ++k) {
    const float inv = 1.0f / smooth[k];
    for (int i = 0; i < M; ++i) amax = std::max(amax, std::fabs(bf16_to_f32(x[(size_t)i * K + k]) * inv));
  }
  *act_scale = amax > 0.f ? amax / 2688.0f : 1.0f;

  // randomized subspace iteration
  std::vector<double> Q((size_t)K * l), Z((size_t)N * l);
  mul_A(W, lam.data(), N, K, omega, l, Q.data());
  orthonormalize(Q.data(), K, l);
  for (int it = 0; it < power_iters; ++it) {
    mul_At(W, lam.data(), N, K, Q.data(), l, Z.data());
    orthonormalize(Z.data(), N, l);
    mul_A(W, lam.data(), N, K, Z.data(), l, Q.data());
    orthonormalize(Q.data(), K, l);
  }
  std::vector<double> Bt((size_t)N * l);  // B^T = A^T Q
  mul_At(W, lam.data(), N, K, Q.data(), l, Bt.data());
  std::vector<double> G((size_t)l * l, 0.0);  // B B^T
  for (int n = 0; n < N; ++n)
    for (int a = 0; a < l; ++a) {
      const double ba = Bt[(size_t)n * l + a];
      for (int c = 0; c < l; ++c) G[(size_t)a * l + c] += ba * Bt[(size_t)n * l + c];
    }
  std::vector<double> E;
  jacobi_eigen(G, l, E);
  std::vector<int> order(l);
  for (int i = 0; i < l; ++i) order[i] = i;
  std::stable_sort(order.begin(), order.end(),
                   [&](int a, int b) { return G[(size_t)a * l + a] > G[(size_t)b * l + b]; });
  for (int t = 0; t < rank; ++t) {
    const int e = order[t];
    const double s = std::sqrt(std::max(G[(size_t)e * l + e], 0.0));
    // U[:, t] = Q Ub[:, e]
    std::vector<double> u(K);
    for (int k = 0; k < K; ++k) {
      double acc = 0.0;
      for (int c = 0; c < l; ++c) acc += Q[(size_t)k * l + c] * E[(size_t)c * l + e];
      u[k] = acc;
    }
    int kmax = 0;
    for (int k = 1; k < K; ++k)
      if (std::fabs(u[k]) > std::fabs(u[kmax])) kmax = k;
    const double sign = u[kmax] < 0 ? -1.0 : 1.0;
    for (int k = 0; k < K; ++k) L1[(size_t)k * rank + t] = f32_to_bf16_rne((float)(sign * u[k] * s));
    // Vt[t, :] = (1/s) Ub[:, e]^T B
    for (int n = 0; n < N; ++n) {
      double acc = 0.0;
      for (int c = 0; c < l; ++c) acc += E[(size_t)c * l + e] * Bt[(size_t)n * l + c];
      L2[(size_t)t * N + n] = f32_to_bf16_rne(s > 0 ? (float)(sign * acc / s) : 0.0f);
    }
  }
  return SVDQ_OK;
}
