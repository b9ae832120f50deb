// Plain single-threaded C++ oracle of the ReSpinQuant block-boundary path.
//
// TEST INFRASTRUCTURE ONLY, like respin_oracle.py: only tests/, the smoke
// check and the benchmark's CPU legs may load it. It shares no code with the
// CUDA library and never calls it; it follows the same readings of the pages
// as respin_oracle.py (ReSpinQuant explainer pages, zh §2.2 steps 1-3 for the
// subspace fix in the row convention, zh §3-§4 and fr §4 for W4A4 / W3A3):
//
//   factors    : the plan's bfloat16 copies of U_r, V_r (round to nearest even)
//   boundary   : h = (residual + x) + (residual U) V^T     in float64, plain loops
//   subspace   : the stored form of zh §2.2 (basis Q, rotation R_sub): the plan
//                holds bfloat16(Q) and M = float(R_sub - I) (difference exact,
//                one rounding to binary32); per token, in float64 and in the
//                page's step order: y = residual Q (projection), z = y M^T
//                (transform inside the subspace), h = residual + x + z Q^T
//                (re-projection and residual)
//   h'         : bfloat16(h), one rounding to nearest even
//   quantizer  : binary32 on g = float(h'): amax = max|g|; amax < 2^-125 gives
//                scale 0 and zero codes; else inv = qmax / amax,
//                q = clamp(rint(g inv), -qmax-1, qmax) (ties to even),
//                scale = amax / qmax, qmax = 7 (INT4) or 3 (INT3)
//   GEMM       : acc[n][o] = sum_k a[n][k] w[o][k] exactly (int64), then
//                bf16((float(acc) * sa[n]) * sw[o]) in binary32
//   packing    : element 2j in the low nibble of byte j, 2j+1 in the high
//                nibble, two's complement
//
// Build: g++ -O2 -std=c++17 -fPIC -shared -ffp-contract=off (no fused
// multiply-add, no fast-math: every float operation is one IEEE rounding).
#include <cfenv>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

namespace {

const float kZeroTokenAmax = 0x1p-125f;
const double kBf16Max = (2.0 - 0x1p-7) * 0x1p127;

// Nearest bfloat16 (ties to even) of a double, as the 16-bit pattern. Normal
// values keep 8 significant bits; below 2^-126 the quantum is 2^-133.
uint16_t bf16_bits_of(double v) {
  if (std::isnan(v)) return 0x7FC0;
  double r = v;
  if (v != 0.0 && std::isfinite(v)) {
    int e = 0;
    std::frexp(v, &e);                       // |v| in [2^(e-1), 2^e)
    const int q = (e < -125 ? -125 : e) - 8;
    r = std::ldexp(std::nearbyint(std::ldexp(v, -q)), q);   // exact scalings, RNE
    if (std::fabs(r) > kBf16Max) r = std::copysign(INFINITY, r);
  }
  const float f = static_cast<float>(r);     // exact: r is a bfloat16 value
  uint32_t u;
  std::memcpy(&u, &f, 4);
  return static_cast<uint16_t>(u >> 16);
}

float bf16_to_float(uint16_t b) {
  const uint32_t u = static_cast<uint32_t>(b) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

// Quantizer of one token (binary32 on the bfloat16-rounded h'): fills hbits,
// h64 (if given), codes and *scale.
void quantize_token(const double* h, int D, int qmax, double* h64, uint16_t* hbits, int8_t* c, float* scale,
                    std::vector<float>& g) {
  const float qm = static_cast<float>(qmax);
  float amax = 0.0f;
  for (int d = 0; d < D; ++d) {
    const uint16_t b = bf16_bits_of(h[d]);
    hbits[d] = b;
    if (h64 != nullptr) h64[d] = h[d];
    g[d] = bf16_to_float(b);
    amax = std::fmax(amax, std::fabs(g[d]));
  }
  if (!(amax >= kZeroTokenAmax)) {
    *scale = 0.0f;
    for (int d = 0; d < D; ++d) c[d] = 0;
    return;
  }
  const float inv = qm / amax;
  for (int d = 0; d < D; ++d) {
    const float t = g[d] * inv;
    float q = std::nearbyint(t);
    if (q > qm) q = qm;
    if (q < -qm - 1.0f) q = -qm - 1.0f;
    c[d] = static_cast<int8_t>(q);
  }
  *scale = amax / qm;
}

int nibble(const uint8_t* row, int k) {
  const int v = (k & 1) ? (row[k >> 1] >> 4) : (row[k >> 1] & 0xF);
  return v >= 8 ? v - 16 : v;
}

}  // namespace

extern "C" {

// One boundary call for N tokens of D channels. x, res: bfloat16 bit patterns
// [N][D] (res may be NULL: zero residual, factors unused). U, V: float [D][r]
// (rounded to bfloat16 here, as the plan does). qmax: 7 or 3. Outputs:
// h64 [N][D] (may be NULL), hbits [N][D], codes [N][D], scale [N].
// Returns 0, or -1 for a bad argument.
int oracle_boundary(int N, int D, int r, const uint16_t* x, const uint16_t* res, const float* U,
                    const float* V, int qmax, double* h64, uint16_t* hbits, int8_t* codes, float* scale) {
  if (N < 0 || D <= 0 || r < 0 || x == nullptr || hbits == nullptr || codes == nullptr || scale == nullptr ||
      (qmax != 7 && qmax != 3) || (res != nullptr && r > 0 && (U == nullptr || V == nullptr)))
    return -1;
  std::fesetround(FE_TONEAREST);
  std::vector<double> Uq(static_cast<size_t>(D) * r), Vq(static_cast<size_t>(D) * r);
  for (size_t i = 0; i < Uq.size(); ++i) {
    Uq[i] = bf16_to_float(bf16_bits_of(U[i]));
    Vq[i] = bf16_to_float(bf16_bits_of(V[i]));
  }
  std::vector<double> h(D), y(r);
  std::vector<float> g(D);
  for (int n = 0; n < N; ++n) {
    const uint16_t* xr = x + static_cast<size_t>(n) * D;
    for (int d = 0; d < D; ++d) h[d] = bf16_to_float(xr[d]);
    if (res != nullptr) {
      const uint16_t* rr = res + static_cast<size_t>(n) * D;
      for (int d = 0; d < D; ++d) h[d] += bf16_to_float(rr[d]);        // residual + x
      for (int j = 0; j < r; ++j) y[j] = 0.0;
      for (int d = 0; d < D; ++d) {                                       // y = residual U
        const double v = bf16_to_float(rr[d]);
        for (int j = 0; j < r; ++j) y[j] += v * Uq[static_cast<size_t>(d) * r + j];
      }
      for (int d = 0; d < D; ++d) {                                       // + y V^T
        double c = 0.0;
        for (int j = 0; j < r; ++j) c += y[j] * Vq[static_cast<size_t>(d) * r + j];
        h[d] += c;
      }
    }
    const size_t o = static_cast<size_t>(n) * D;
    quantize_token(h.data(), D, qmax, h64 != nullptr ? h64 + o : nullptr, hbits + o, codes + o, scale + n, g);
  }
  return 0;
}

// The same call with the plan in the stored subspace form: Q float [D][r],
// R_sub float [r][r] (row-major). Plan values: bfloat16(Q) and
// M = float(R_sub - I). Returns 0, or -1 for a bad argument.
int oracle_boundary_subspace(int N, int D, int r, const uint16_t* x, const uint16_t* res, const float* Q,
                             const float* R_sub, int qmax, double* h64, uint16_t* hbits, int8_t* codes,
                             float* scale) {
  if (N < 0 || D <= 0 || r < 0 || x == nullptr || hbits == nullptr || codes == nullptr || scale == nullptr ||
      (qmax != 7 && qmax != 3) || (res != nullptr && r > 0 && (Q == nullptr || R_sub == nullptr)))
    return -1;
  std::fesetround(FE_TONEAREST);
  std::vector<double> Qq(static_cast<size_t>(D) * r), M(static_cast<size_t>(r) * r);
  for (size_t i = 0; i < Qq.size(); ++i) Qq[i] = bf16_to_float(bf16_bits_of(Q[i]));
  for (int i = 0; i < r; ++i)
    for (int j = 0; j < r; ++j) {
      const double d = static_cast<double>(R_sub[static_cast<size_t>(i) * r + j]) - (i == j ? 1.0 : 0.0);
      M[static_cast<size_t>(i) * r + j] = static_cast<double>(static_cast<float>(d));
    }
  std::vector<double> h(D), y(r), z(r);
  std::vector<float> g(D);
  for (int n = 0; n < N; ++n) {
    const uint16_t* xr = x + static_cast<size_t>(n) * D;
    for (int d = 0; d < D; ++d) h[d] = bf16_to_float(xr[d]);
    if (res != nullptr) {
      const uint16_t* rr = res + static_cast<size_t>(n) * D;
      for (int d = 0; d < D; ++d) h[d] += bf16_to_float(rr[d]);        // residual + x
      for (int j = 0; j < r; ++j) y[j] = 0.0;
      for (int d = 0; d < D; ++d) {                                       // step 1: y = residual Q
        const double v = bf16_to_float(rr[d]);
        for (int j = 0; j < r; ++j) y[j] += v * Qq[static_cast<size_t>(d) * r + j];
      }
      for (int i = 0; i < r; ++i) {                                       // step 2: z = y M^T
        double a = 0.0;
        for (int j = 0; j < r; ++j) a += y[j] * M[static_cast<size_t>(i) * r + j];
        z[i] = a;
      }
      for (int d = 0; d < D; ++d) {                                       // step 3: + z Q^T
        double c = 0.0;
        for (int i = 0; i < r; ++i) c += z[i] * Qq[static_cast<size_t>(d) * r + i];
        h[d] += c;
      }
    }
    const size_t o = static_cast<size_t>(n) * D;
    quantize_token(h.data(), D, qmax, h64 != nullptr ? h64 + o : nullptr, hbits + o, codes + o, scale + n, g);
  }
  return 0;
}

// Packing of codes [rows][K] (K even) into [rows][K/2].
int oracle_pack(int rows, int K, const int8_t* codes, uint8_t* packed) {
  if (rows < 0 || K <= 0 || K % 2 || codes == nullptr || packed == nullptr) return -1;
  for (int i = 0; i < rows; ++i)
    for (int j = 0; j < K / 2; ++j) {
      const int lo = codes[static_cast<size_t>(i) * K + 2 * j] & 0xF;
      const int hi = codes[static_cast<size_t>(i) * K + 2 * j + 1] & 0xF;
      packed[static_cast<size_t>(i) * (K / 2) + j] = static_cast<uint8_t>(lo | (hi << 4));
    }
  return 0;
}

// W4A4 (or W3A3) GEMM: qa [N][K/2], qw [O][K/2] packed codes; sa [N], sw [O].
// acc [N][O] exact; outbits [N][O] bfloat16 of the binary32 epilogue (may be
// NULL, then sa and sw may be NULL too). Returns 0, -1 for a bad argument,
// -2 if an accumulator is not exact in binary32 (|acc| >= 2^24).
int oracle_w4a4(int N, int K, int O, const uint8_t* qa, const float* sa, const uint8_t* qw, const float* sw,
                int64_t* acc, uint16_t* outbits) {
  if (N < 0 || K <= 0 || K % 2 || O <= 0 || qa == nullptr || qw == nullptr || acc == nullptr ||
      (outbits != nullptr && (sa == nullptr || sw == nullptr)))
    return -1;
  std::fesetround(FE_TONEAREST);
  std::vector<int8_t> w(static_cast<size_t>(O) * K);   // the weight codes, unpacked once
  for (int o = 0; o < O; ++o)
    for (int k = 0; k < K; ++k) w[static_cast<size_t>(o) * K + k] = static_cast<int8_t>(nibble(qw + static_cast<size_t>(o) * (K / 2), k));
  std::vector<int> a(K);
  int status = 0;
  for (int n = 0; n < N; ++n) {
    const uint8_t* ar = qa + static_cast<size_t>(n) * (K / 2);
    for (int k = 0; k < K; ++k) a[k] = nibble(ar, k);
    for (int o = 0; o < O; ++o) {
      const int8_t* wr = &w[static_cast<size_t>(o) * K];
      int64_t s = 0;
      for (int k = 0; k < K; ++k) s += static_cast<int64_t>(a[k]) * wr[k];
      acc[static_cast<size_t>(n) * O + o] = s;
      if (outbits != nullptr) {
        if (s >= (int64_t(1) << 24) || s <= -(int64_t(1) << 24)) status = -2;
        const float t = (static_cast<float>(s) * sa[n]) * sw[o];
        outbits[static_cast<size_t>(n) * O + o] = bf16_bits_of(static_cast<double>(t));
      }
    }
  }
  return status;
}

}  // extern "C"
