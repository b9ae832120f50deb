// W4A4 GEMM for few tokens (decode, N <= 128): the same contraction and
// epilogue as w4a4_gemm_kernel,
//
//   acc[n, o] = sum_k a[n, k] w[o, k]            (exact, int32)
//   out[n, o] = bf16((float(acc) * sa[n]) * sw[o])
//
// (W4A4 linear layers of the ReSpinQuant explainers, zh §3-§4, fr §4), laid
// out for the case where the weights are the only large operand: with N
// tokens the contraction does 4 N integer operations per weight byte, so up
// to about a hundred tokens the weight stream from HBM is the bound, and
// every SM must pull its share of it. A 256-token tensor-core tile leaves
// most SMs idle there (O / 256 tiles).
//
// Design:
//  * a CTA owns 16 output channels (O / 16 CTAs) and splits K over KG warp
//    groups (8 / TG warps each way) and the tokens over TG groups of 8 NT;
//  * each warp streams its channels' packed weight rows straight into
//    registers (16-byte non-allocating loads, DEPTH chunks of 128 codes in
//    flight) together with the matching activation chunks (L2-resident,
//    shared by all CTAs), and contracts them on mma.sync m16n8k32 (s8, s32
//    accumulate): channels are the M side, tokens the N side;
//  * INT4 is widened in registers with the nibble-high form used by the
//    tensor-memory kernel: byte = 16 c, one AND (odd codes) or SHIFT + AND
//    (even codes) per 4 bytes. Lane (g, q) takes bytes [16 q, 16 q + 16) of a
//    64-byte chunk; for MMA j of the chunk the even codes of its word j fill
//    the k slots 4q..4q+3 and the odd codes the slots 16+4q..16+4q+3. A and
//    B use the same assignment, so the dot product over k is unchanged; the
//    MMA sums 256 acc exactly (|256 acc| <= 2^14 K < 2^31 for K <= 65536);
//  * the KG partial sums of a CTA are added in shared memory (integer sums:
//    exact and order-free), shifted back by 8 bits and scaled.
// No global scratch, no waits beyond __syncthreads.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

namespace respin {

constexpr int kSkRows = 16;      // output channels per CTA
constexpr int kSkWarps = 8;
constexpr int kSkThreads = 32 * kSkWarps;
constexpr int kSkChunkBytes = 64;  // 128 codes of one row
constexpr int kSkDepth = 4;      // chunks in flight per warp

__device__ __forceinline__ uint4 ldg_nc_na_u4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint32_t sk_word(const uint4& v, int j) {
  return j == 0 ? v.x : j == 1 ? v.y : j == 2 ? v.z : v.w;
}

// even codes of a packed word -> 4 bytes 16 c (codes 0, 2, 4, 6)
__device__ __forceinline__ uint32_t widen_even(uint32_t x) { return (x << 4) & 0xF0F0F0F0u; }
// odd codes -> 4 bytes 16 c (codes 1, 3, 5, 7)
__device__ __forceinline__ uint32_t widen_odd(uint32_t x) { return x & 0xF0F0F0F0u; }

__device__ __forceinline__ void mma_s8_16832(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                             uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// NT n8 token tiles per warp, TG token groups per CTA (tokens per CTA =
// 8 NT TG >= N). qa: [N, K/2], qw: [O, K/2] packed codes; out: bf16 or int32
// [N, O]. Grid: O / 16 CTAs of 256 threads.
template <int NT, int TG, bool I32OUT>
__global__ void __launch_bounds__(kSkThreads, 2)
w4a4_gemm_skinny_kernel(const uint8_t* __restrict__ qa, const float* __restrict__ sa,
                        const uint8_t* __restrict__ qw, const float* __restrict__ sw, int N, int K, int O,
                        void* __restrict__ out) {
  constexpr int KG = kSkWarps / TG;      // K groups
  constexpr int TPG = 8 * NT;            // tokens per group
  constexpr int TOK = TPG * TG;          // tokens per CTA
  constexpr int PP = kSkRows + 1;        // padded channel pitch of the partials
  __shared__ int part[KG][TOK][PP];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, q = lane & 3;
  const int kg = warp % KG, tg = warp / KG;
  const int o0 = blockIdx.x * kSkRows;
  const int KC = K / 128;
  const size_t rowb = static_cast<size_t>(K) / 2;
  const uint8_t* wa = qw + static_cast<size_t>(o0 + g) * rowb + 16 * q;  // channel o0 + g
  const uint8_t* wb = wa + 8 * rowb;                                       // channel o0 + g + 8
  const uint8_t* ab[NT];
  bool av[NT];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int n = tg * TPG + nt * 8 + g;
    av[nt] = n < N;
    ab[nt] = qa + static_cast<size_t>(av[nt] ? n : 0) * rowb + 16 * q;
  }

  int acc[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0;

  for (int c0 = kg; c0 < KC; c0 += KG * kSkDepth) {
    uint4 A0[kSkDepth], A1[kSkDepth];
#pragma unroll
    for (int d = 0; d < kSkDepth; ++d) {
      const int c = c0 + d * KG;
      if (c < KC) {
        A0[d] = ldg_nc_na_u4(wa + static_cast<size_t>(c) * kSkChunkBytes);
        A1[d] = ldg_nc_na_u4(wb + static_cast<size_t>(c) * kSkChunkBytes);
      } else {
        A0[d] = A1[d] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
#pragma unroll
    for (int d = 0; d < kSkDepth; ++d) {
      const int c = c0 + d * KG;
      if (c >= KC) break;  // warp-uniform
      uint4 B[NT];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
        B[nt] = av[nt] ? __ldg(reinterpret_cast<const uint4*>(ab[nt] + static_cast<size_t>(c) * kSkChunkBytes))
                       : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t w0 = sk_word(A0[d], j), w1 = sk_word(A1[d], j);
        const uint32_t a0 = widen_even(w0), a1 = widen_even(w1), a2 = widen_odd(w0), a3 = widen_odd(w1);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const uint32_t bw = sk_word(B[nt], j);
          mma_s8_16832(acc[nt], a0, a1, a2, a3, widen_even(bw), widen_odd(bw));
        }
      }
    }
  }

  // partials: acc[nt] = (channel g, tokens 2q, 2q+1), (channel g + 8, same)
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int n = tg * TPG + nt * 8 + 2 * q;
    part[kg][n][g] = acc[nt][0];
    part[kg][n + 1][g] = acc[nt][1];
    part[kg][n][g + 8] = acc[nt][2];
    part[kg][n + 1][g + 8] = acc[nt][3];
  }
  __syncthreads();

  // outputs: thread -> (channel tid % 16, tokens tid / 16 + 16 i)
  const int oc = tid % kSkRows;
  const int o = o0 + oc;
  float swo = 0.f;
  if constexpr (!I32OUT) swo = sw[o];
  for (int n = tid / kSkRows; n < TOK && n < N; n += kSkThreads / kSkRows) {
    int s = 0;
#pragma unroll
    for (int k = 0; k < KG; ++k) s += part[k][n][oc];
    const int v = s >> 8;  // exact: every partial is a multiple of 256
    if constexpr (I32OUT) {
      static_cast<int32_t*>(out)[static_cast<size_t>(n) * O + o] = v;
    } else {
      const float f = __fmul_rn(__fmul_rn(static_cast<float>(v), sa[n]), swo);
      static_cast<__nv_bfloat16*>(out)[static_cast<size_t>(n) * O + o] = __float2bfloat16_rn(f);
    }
  }
}

}  // namespace respin
