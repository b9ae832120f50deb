// Host-side offline weight preparation (float64 arithmetic, no device):
//
//  * Rotation fusion. The explainers fold each block's learned rotation into
//    the weights of the linears before inference (zh §2.2 "offline weight
//    merging", e.g. W~ = R^T W R; fr §2A, W~ = W R), so that the linears stay
//    ordinary linears. For a linear y = W x whose input arrives in the rotated
//    basis x~ = R_in^T x and whose output is wanted in the basis
//    y~ = R_out^T y:  W~ = R_out^T W R_in,  W~ x~ = R_out^T W x.
//    Without an output rotation, W~ = W R_in.
//  * Weight quantization: symmetric round-to-nearest per output channel (one
//    fp32 scale per row), the same binary32 quantizer as the activations:
//    amax = max |w|, inv = qmax / amax, q = clamp(rint(w inv), -qmax-1, qmax),
//    scale = amax / qmax (qmax = 7 for INT4, 3 for INT3), codes packed two per
//    byte (element 2j in the low nibble).
//
// The products are blocked and spread over host threads (std::thread); every
// output element is one float64 sum in a fixed order, so the result does not
// depend on the thread count.
#pragma once

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <thread>
#include <vector>

namespace respin {
namespace host {

// C (m x n) = op(A) (m x k) * B (k x n), all row-major float64; op(A) = A or
// A^T (A stored k x m). Rows of C are split over threads; within a row block
// the k loop is tiled so that a tile of B stays in cache.
inline void dgemm_rows(int m, int n, int k, const double* A, bool transA, const double* B, double* C) {
  const int nthreads = std::max(1u, std::min(64u, std::thread::hardware_concurrency()));
  const int rb = 16, kb = 128;
  auto work = [&](int t) {
    std::vector<double> acc(static_cast<size_t>(rb) * n);
    for (int i0 = t * rb; i0 < m; i0 += nthreads * rb) {
      const int ir = std::min(rb, m - i0);
      std::fill(acc.begin(), acc.end(), 0.0);
      for (int k0 = 0; k0 < k; k0 += kb) {
        const int kr = std::min(kb, k - k0);
        for (int i = 0; i < ir; ++i) {
          double* c = &acc[static_cast<size_t>(i) * n];
          for (int kk = 0; kk < kr; ++kk) {
            const int kx = k0 + kk;
            const double a = transA ? A[static_cast<size_t>(kx) * m + i0 + i] : A[static_cast<size_t>(i0 + i) * k + kx];
            if (a == 0.0) continue;
            const double* b = &B[static_cast<size_t>(kx) * n];
            for (int j = 0; j < n; ++j) c[j] += a * b[j];
          }
        }
      }
      std::copy(acc.begin(), acc.begin() + static_cast<size_t>(ir) * n, C + static_cast<size_t>(i0) * n);
    }
  };
  std::vector<std::thread> pool;
  for (int t = 1; t < nthreads; ++t) pool.emplace_back(work, t);
  work(0);
  for (auto& th : pool) th.join();
}

// W_fused (O x K) = R_out^T W R_in (R_out may be null: W R_in). W, R_in,
// R_out: float32 row-major (O x K, K x K, O x O). Returns false on bad sizes.
inline bool fuse_weight(int O, int K, const float* W, const float* R_in, const float* R_out, float* W_fused) {
  if (O <= 0 || K <= 0 || W == nullptr || R_in == nullptr || W_fused == nullptr) return false;
  std::vector<double> w(W, W + static_cast<size_t>(O) * K), r(R_in, R_in + static_cast<size_t>(K) * K);
  std::vector<double> t(static_cast<size_t>(O) * K);
  dgemm_rows(O, K, K, w.data(), false, r.data(), t.data());   // W R_in
  if (R_out != nullptr) {
    std::vector<double> ro(R_out, R_out + static_cast<size_t>(O) * O);
    dgemm_rows(O, K, O, ro.data(), true, t.data(), w.data());  // R_out^T (W R_in)
    t.swap(w);
  }
  for (size_t i = 0; i < t.size(); ++i) W_fused[i] = static_cast<float>(t[i]);
  return true;
}

// Per-row symmetric quantization of W (O x K float32, K even) with bound
// qmax (7 or 3): packed codes q_w (O x K/2) and scales (O).
inline bool quantize_weight_rows(int O, int K, const float* W, int qmax, uint8_t* q_w, float* scale) {
  if (O <= 0 || K <= 0 || K % 2 || W == nullptr || q_w == nullptr || scale == nullptr || (qmax != 7 && qmax != 3))
    return false;
  const float qm = static_cast<float>(qmax);
  const float zero_amax = 2.3509887e-38f;   // 2^-125: below it qmax / amax overflows binary32
  for (int o = 0; o < O; ++o) {
    const float* w = W + static_cast<size_t>(o) * K;
    float amax = 0.0f;
    for (int k = 0; k < K; ++k) amax = std::fmax(amax, std::fabs(w[k]));
    uint8_t* qo = q_w + static_cast<size_t>(o) * (K / 2);
    if (!(amax >= zero_amax)) {
      scale[o] = 0.0f;
      for (int j = 0; j < K / 2; ++j) qo[j] = 0;
      continue;
    }
    const volatile float inv = qm / amax;   // one binary32 division, kept apart from the products
    auto code = [&](float v) {
      const volatile float t = v * inv;
      float q = std::nearbyint(static_cast<float>(t));
      q = std::fmin(std::fmax(q, -qm - 1.0f), qm);
      return static_cast<int>(q) & 0xF;
    };
    for (int j = 0; j < K / 2; ++j) qo[j] = static_cast<uint8_t>(code(w[2 * j]) | (code(w[2 * j + 1]) << 4));
    scale[o] = amax / qm;
  }
  return true;
}

}  // namespace host
}  // namespace respin
