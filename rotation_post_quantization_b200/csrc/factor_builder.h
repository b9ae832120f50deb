// Host-side builders of the rank-r boundary factors (offline, float64).
//
// The boundary fix is h' = residual (I + U_r V_r^T) + x (row convention).
//  * From the subspace form of the ReSpinQuant explainers (zh §2.2 steps 1-3:
//    y = Q^T x, M = R_sub - I, x_out = x + Q (M y) for a column vector):
//    with h = x^T the same map is h + (h Q) (Q M)^T, so U_r = Q, V_r = Q M.
//  * From a dense transition T (it §2C, nl §2C, es §2B, fr §2C: the top-r
//    SVD of Delta T = T - I gives the subspace): in the row convention
//    h' = h T, so with Delta T = sum_i s_i u_i v_i^T the rank-r fix is
//    h U_r V_r^T with U_r = [u_1 .. u_r] and V_r = [s_1 v_1 .. s_r v_r].
//    The leading singular triplets come from block subspace iteration in
//    float64 (Halko, Martinsson and Tropp, "Finding structure with
//    randomness", 2011: range finder with power iterations, then the SVD of
//    the small projected matrix), the small symmetric eigenproblem from cyclic
//    Jacobi rotations. The truncation is refused when s_r and s_(r+1) are too
//    close for the top-r subspace to be well defined.
#pragma once

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <vector>

namespace respin {
namespace host {

// Modified Gram-Schmidt, twice, on the k columns of Y (n x k row-major).
// Returns false if a column is numerically dependent on the previous ones.
inline bool orthonormalize_columns(std::vector<double>& Y, int n, int k) {
  for (int pass = 0; pass < 2; ++pass) {
    for (int j = 0; j < k; ++j) {
      for (int i = 0; i < j; ++i) {
        double dot = 0.0;
        for (int t = 0; t < n; ++t) dot += Y[static_cast<size_t>(t) * k + i] * Y[static_cast<size_t>(t) * k + j];
        for (int t = 0; t < n; ++t) Y[static_cast<size_t>(t) * k + j] -= dot * Y[static_cast<size_t>(t) * k + i];
      }
      double nrm = 0.0;
      for (int t = 0; t < n; ++t) nrm += Y[static_cast<size_t>(t) * k + j] * Y[static_cast<size_t>(t) * k + j];
      nrm = std::sqrt(nrm);
      if (!(nrm > 1e-300)) return false;
      for (int t = 0; t < n; ++t) Y[static_cast<size_t>(t) * k + j] /= nrm;
    }
  }
  return true;
}

// out (n x k) = A (n x n, row-major) * Y (n x k), or A^T * Y if transpose.
inline void mat_block(const std::vector<double>& A, int n, const std::vector<double>& Y, int k,
                      std::vector<double>& out, bool transpose) {
  out.assign(static_cast<size_t>(n) * k, 0.0);
  for (int a = 0; a < n; ++a)
    for (int b = 0; b < n; ++b) {
      const double v = transpose ? A[static_cast<size_t>(b) * n + a] : A[static_cast<size_t>(a) * n + b];
      if (v == 0.0) continue;
      const double* y = &Y[static_cast<size_t>(b) * k];
      double* o = &out[static_cast<size_t>(a) * k];
      for (int j = 0; j < k; ++j) o[j] += v * y[j];
    }
}

// Eigen-decomposition of the symmetric k x k matrix S (row-major) by cyclic
// Jacobi rotations: on return S is diagonal (the eigenvalues) and E holds the
// eigenvectors as columns.
inline void jacobi_eigen(std::vector<double>& S, int k, std::vector<double>& E) {
  E.assign(static_cast<size_t>(k) * k, 0.0);
  for (int i = 0; i < k; ++i) E[static_cast<size_t>(i) * k + i] = 1.0;
  for (int sweep = 0; sweep < 100; ++sweep) {
    double off = 0.0, diag = 0.0;
    for (int i = 0; i < k; ++i)
      for (int j = 0; j < k; ++j) {
        const double v = S[static_cast<size_t>(i) * k + j];
        (i == j ? diag : off) += v * v;
      }
    if (off <= 1e-30 * diag || off == 0.0) break;
    for (int p = 0; p < k - 1; ++p)
      for (int q = p + 1; q < k; ++q) {
        const double apq = S[static_cast<size_t>(p) * k + q];
        if (apq == 0.0) continue;
        const double app = S[static_cast<size_t>(p) * k + p], aqq = S[static_cast<size_t>(q) * k + q];
        const double theta = (aqq - app) / (2.0 * apq);
        const double t = (theta >= 0 ? 1.0 : -1.0) / (std::fabs(theta) + std::sqrt(theta * theta + 1.0));
        const double c = 1.0 / std::sqrt(t * t + 1.0), s = t * c;
        for (int i = 0; i < k; ++i) {   // S <- S J (columns p, q)
          const double sip = S[static_cast<size_t>(i) * k + p], siq = S[static_cast<size_t>(i) * k + q];
          S[static_cast<size_t>(i) * k + p] = c * sip - s * siq;
          S[static_cast<size_t>(i) * k + q] = s * sip + c * siq;
        }
        for (int j = 0; j < k; ++j) {   // S <- J^T S (rows p, q)
          const double spj = S[static_cast<size_t>(p) * k + j], sqj = S[static_cast<size_t>(q) * k + j];
          S[static_cast<size_t>(p) * k + j] = c * spj - s * sqj;
          S[static_cast<size_t>(q) * k + j] = s * spj + c * sqj;
        }
        for (int i = 0; i < k; ++i) {   // E <- E J
          const double eip = E[static_cast<size_t>(i) * k + p], eiq = E[static_cast<size_t>(i) * k + q];
          E[static_cast<size_t>(i) * k + p] = c * eip - s * eiq;
          E[static_cast<size_t>(i) * k + q] = s * eip + c * eiq;
        }
      }
  }
}

// xorshift64* stream in [-1, 1): the starting block of the range finder.
inline double start_value(uint64_t& state) {
  state ^= state >> 12;
  state ^= state << 25;
  state ^= state >> 27;
  const uint64_t v = state * 0x2545F4914F6CDD1DULL;
  return static_cast<double>(v >> 11) * (2.0 / 9007199254740992.0) - 1.0;
}

enum class BuildResult { kOk, kBadArg, kNoGap, kNoConvergence };

// Top-r factors of Delta T = T - I (T: n x n row-major, float). sigma_out
// (may be NULL) receives s_1 .. s_(r+1) (0 past the block). gap_tol: the
// truncation is refused unless s_r - s_(r+1) > gap_tol * s_1.
inline BuildResult factors_from_transition(int n, int r, const float* T, double gap_tol, float* U_out,
                                           float* V_out, double* sigma_out) {
  if (n <= 0 || r <= 0 || r >= n || T == nullptr || U_out == nullptr || V_out == nullptr) return BuildResult::kBadArg;
  std::vector<double> A(static_cast<size_t>(n) * n);
  for (int i = 0; i < n; ++i)
    for (int j = 0; j < n; ++j)
      A[static_cast<size_t>(i) * n + j] = static_cast<double>(T[static_cast<size_t>(i) * n + j]) - (i == j ? 1.0 : 0.0);
  const int k = std::min(n, std::max(2 * r, r + 8));   // block: r plus oversampling
  std::vector<double> Y(static_cast<size_t>(n) * k), Z, B, S, E, Vr, Vprev;
  uint64_t st = 0x9E3779B97F4A7C15ULL;
  for (auto& v : Y) v = start_value(st);
  if (!orthonormalize_columns(Y, n, k)) return BuildResult::kNoConvergence;
  std::vector<double> sig(k, 0.0);
  std::vector<int> order(k);
  bool converged = false;
  for (int it = 0; it < 300 && !converged; ++it) {
    // Rayleigh-Ritz on the block Y (orthonormal, n x k): with B = A Y the
    // eigenpairs (s^2, e) of B^T B give right singular vectors v = Y e and
    // left ones u = B e / s
    mat_block(A, n, Y, k, B, false);
    S.assign(static_cast<size_t>(k) * k, 0.0);
    for (int a = 0; a < k; ++a)
      for (int b = a; b < k; ++b) {
        double sum = 0.0;
        for (int t = 0; t < n; ++t) sum += B[static_cast<size_t>(t) * k + a] * B[static_cast<size_t>(t) * k + b];
        S[static_cast<size_t>(a) * k + b] = S[static_cast<size_t>(b) * k + a] = sum;
      }
    jacobi_eigen(S, k, E);
    for (int i = 0; i < k; ++i) {
      sig[i] = std::sqrt(std::max(0.0, S[static_cast<size_t>(i) * k + i]));
      order[i] = i;
    }
    std::sort(order.begin(), order.end(), [&](int a, int b) { return sig[a] > sig[b]; });
    if (!(sig[order[0]] > 0.0)) break;   // Delta T = 0 on the block: no gap (below)
    // the top-r Ritz vectors; converged once their span stops moving
    Vr.assign(static_cast<size_t>(n) * r, 0.0);
    for (int t = 0; t < n; ++t)
      for (int c = 0; c < r; ++c) {
        double v = 0.0;
        for (int j = 0; j < k; ++j) v += Y[static_cast<size_t>(t) * k + j] * E[static_cast<size_t>(j) * k + order[c]];
        Vr[static_cast<size_t>(t) * r + c] = v;
      }
    if (!Vprev.empty()) {
      // || Vr - Vprev (Vprev^T Vr) ||_F
      std::vector<double> P(static_cast<size_t>(r) * r, 0.0);
      for (int a = 0; a < r; ++a)
        for (int b = 0; b < r; ++b) {
          double sum = 0.0;
          for (int t = 0; t < n; ++t) sum += Vprev[static_cast<size_t>(t) * r + a] * Vr[static_cast<size_t>(t) * r + b];
          P[static_cast<size_t>(a) * r + b] = sum;
        }
      double res = 0.0;
      for (int t = 0; t < n; ++t)
        for (int b = 0; b < r; ++b) {
          double v = Vr[static_cast<size_t>(t) * r + b];
          for (int a = 0; a < r; ++a) v -= Vprev[static_cast<size_t>(t) * r + a] * P[static_cast<size_t>(a) * r + b];
          res += v * v;
        }
      converged = std::sqrt(res) <= 1e-12 * std::sqrt(static_cast<double>(r));
    }
    Vprev = Vr;
    if (converged) break;
    // one power step on the right singular subspace: Y <- orth(A^T orth(A Y))
    Z = B;
    if (!orthonormalize_columns(Z, n, k)) return BuildResult::kNoConvergence;
    mat_block(A, n, Z, k, Y, true);
    if (!orthonormalize_columns(Y, n, k)) return BuildResult::kNoConvergence;
  }
  const double s1 = sig[order[0]];
  const double sr = sig[order[r - 1]], sr1 = r < k ? sig[order[r]] : 0.0;
  if (sigma_out != nullptr)
    for (int i = 0; i <= r; ++i) sigma_out[i] = i < k ? sig[order[i]] : 0.0;
  // without a gap the top-r subspace is not unique (and does not settle)
  if (!(s1 > 0.0) || !(sr - sr1 > gap_tol * s1)) return BuildResult::kNoGap;
  if (!converged) return BuildResult::kNoConvergence;
  // Delta T = sum_i s_i u_i v_i^T, so h Delta T_r = (h U_r) V_r^T with
  // U_r = [u_i] and V_r = [s_i v_i]
  for (int c = 0; c < r; ++c) {
    const int e = order[c];
    const double s = sig[e];
    for (int t = 0; t < n; ++t) {
      double bu = 0.0;
      for (int j = 0; j < k; ++j) bu += B[static_cast<size_t>(t) * k + j] * E[static_cast<size_t>(j) * k + e];
      U_out[static_cast<size_t>(t) * r + c] = static_cast<float>(bu / s);
      V_out[static_cast<size_t>(t) * r + c] = static_cast<float>(s * Vr[static_cast<size_t>(t) * r + c]);
    }
  }
  return BuildResult::kOk;
}

// U_r = Q, V_r = Q (R_sub - I): Q is n x r row-major, R_sub r x r row-major.
inline BuildResult factors_from_subspace(int n, int r, const float* Q, const float* R_sub, float* U_out,
                                         float* V_out) {
  if (n <= 0 || r <= 0 || r > n || Q == nullptr || R_sub == nullptr || U_out == nullptr || V_out == nullptr)
    return BuildResult::kBadArg;
  for (int t = 0; t < n; ++t)
    for (int c = 0; c < r; ++c) {
      U_out[static_cast<size_t>(t) * r + c] = Q[static_cast<size_t>(t) * r + c];
      double v = 0.0;
      for (int j = 0; j < r; ++j) {
        const double m = static_cast<double>(R_sub[static_cast<size_t>(j) * r + c]) - (j == c ? 1.0 : 0.0);
        v += static_cast<double>(Q[static_cast<size_t>(t) * r + j]) * m;
      }
      V_out[static_cast<size_t>(t) * r + c] = static_cast<float>(v);
    }
  return BuildResult::kOk;
}

}  // namespace host
}  // namespace respin
